// k_phi.cuh -- token compression phi (page "硬件对齐+原生训练！DeepSeek NSA打造高效
// 稀疏Attention", 令牌压缩; explainer "DeepseekNativelySparseAttention", 2.2-2.3) and
// the layout helpers the attention kernels read.
//
//   mean:   K~[i] = (1/l) sum_j k[i*d + j]
//   linear: K~[i] = W vec(k_blk + E) = W vec(k_blk) + W vec(E)
//           vec is position-major: x[j*D + c] = k[i*d + j][c] + E[j][c].
// The linear map is a GEMM [C x l*D] x [l*D x D] on tcgen05 (bf16 in, fp32
// accumulate in TMEM); the constant W vec(E) is precomputed in fp64 and added
// in the epilogue.  Outputs are bf16 (round to nearest even): K~ as
// [B,C,G,dk] and V~ transposed as [B,G,dv,Cp] for the P.V~ products (plus
// V~ as [B,C,G,dv] when the caller asks for it).
//
// Correct rounding.  The GEMM accumulates chunks of 256 products in fp32 on
// the tensor cores and sums the chunks in fp64, so the value before rounding
// is off only by the fp32 rounding of chunk partial sums.  An element whose
// value lies within kPhiMargin (+ 2^-16 relative) of a bf16 rounding midpoint
// -- a bound well above that error -- could still round to the wrong
// neighbour: the epilogue lists those elements and phi_fixup_kernel
// recomputes them exactly in fp64 and rounds them once.  The result is the
// correctly rounded bf16 of W vec(k_blk + E).
#pragma once
#include "nsa_dev.cuh"
#include "k_attn_packed.cuh"   // wait_or_abort

namespace nsa {

// fp64 -> bf16, round to nearest even in one step: round to odd into fp32
// (24 bits), then nearest-even into bf16 (8 bits).  Round-to-odd with at least
// two extra bits makes the second rounding exact.
__device__ __forceinline__ __nv_bfloat16 d2bf16_rn(double x) {
    float f = __double2float_rz(x);
    if ((double)f != x) {
        uint32_t u = __float_as_uint(f) | 1u;
        f = __uint_as_float(u);
    }
    return __float2bfloat16_rn(f);
}

// ---------------------------------------------------------------- mean phi
// grid (C, G, B), block 256.  fp64 accumulation of l bf16 values is exact,
// so the result is the correctly rounded mean.
__global__ void phi_mean_kernel(const __nv_bfloat16* __restrict__ x, int T, int G, int D, int l,
                                int d, int C, int Cp, __nv_bfloat16* __restrict__ y,
                                __nv_bfloat16* __restrict__ yT) {
    const int i = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
        double acc = 0.0;
        const __nv_bfloat16* src = x + (((size_t)b * T + (size_t)i * d) * G + g) * D + c;
        for (int j = 0; j < l; ++j) acc += (double)__bfloat162float(src[(size_t)j * G * D]);
        __nv_bfloat16 r = d2bf16_rn(acc / (double)l);
        if (y) y[(((size_t)b * C + i) * G + g) * D + c] = r;
        if (yT) yT[(((size_t)b * G + g) * D + c) * Cp + i] = r;
    }
}

// --------------------------------------------------------- linear phi bias
// bias[o] = sum_x W[o, x] * E_flat[x] in fp64.  grid D, block 256.
__global__ void phi_bias_kernel(const __nv_bfloat16* __restrict__ W,
                                const __nv_bfloat16* __restrict__ E, int K, double* __restrict__ bias) {
    __shared__ double red[256];
    const int o = blockIdx.x;
    double acc = 0.0;
    for (int x = threadIdx.x; x < K; x += blockDim.x)
        acc += (double)__bfloat162float(W[(size_t)o * K + x]) * (double)__bfloat162float(E[x]);
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int s = blockDim.x / 2; s > 0; s >>= 1) {
        if ((int)threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0) bias[o] = red[0];
}

// ------------------------------------------------------- linear phi (GEMM)
// One CTA computes 128 compressed blocks x NH = D/2 outputs for one
// (group, output half, batch).  Warps 0-3: epilogue (thread = row).  Warp 4:
// TMA producer.  Warp 5: MMA issuer and TMEM owner.
//   A (K-step (j, cc)): rows i0..i0+127 of token (i + j/d)*d + j%d, channels
//      cc*64..+63, through a 5-D map {D, G, d, floor(T/d), B}.
//   B: W[half*NH .. +NH, j*D + cc*64 .. +63] through a 2-D map {l*D, D}.
// The K loop runs in chunks of kPhiChunk K-steps (256 products per output);
// each chunk accumulates in fp32 in one of two TMEM buffers and the epilogue
// folds it into fp64 accumulators in shared memory while the next chunk runs.
// The fp32 rounding error therefore only involves chunk-sized partial sums.
constexpr int kPhiChunk = 4;                  // K-steps of 64 per chunk
constexpr float kPhiMargin = 1.0f / 16384.0f; // absolute, in the units of K~

template <int D>
struct PhiGemmCfg {
    static constexpr int NH = D / 2;
    static constexpr int kStages = 4;
    static constexpr int kABytes = 128 * 128;          // 128 rows x 64 bf16
    static constexpr int kBBytes = NH * 128;           // NH rows x 64 bf16
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kAccBytes = NH * 128 * 8;     // fp64 [NH][128]
    static constexpr int kSmem = kStages * kStageBytes + kAccBytes + 1024 /*align*/ + 256 /*barriers*/;
    static constexpr uint32_t kTmemCols = 2 * NH <= 64 ? 64 : (2 * NH <= 128 ? 128 : 256);
};

// true when v lies within the margin of a bf16 rounding midpoint
__device__ __forceinline__ bool near_bf16_midpoint(double v) {
    if (fabs(v) < 1e-30) return true;
    const __nv_bfloat16 r = d2bf16_rn(v);
    const double rv = (double)__bfloat162float(r);
    // neighbour in the direction of v and the midpoint between the two
    const uint16_t bits = *reinterpret_cast<const uint16_t*>(&r);
    const uint16_t nb = (v > rv) == (rv >= 0.0) ? (uint16_t)(bits + 1) : (uint16_t)(bits - 1);
    const double nv = (double)__bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(&nb));
    const double mid = 0.5 * (rv + nv);
    return fabs(v - mid) <= (double)kPhiMargin + fabs(v) * (1.0 / 65536.0);
}

template <int D>
__global__ void __launch_bounds__(192, 1)
    phi_linear_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapW,
                      const double* __restrict__ bias, int l, int d, int C, int Cp, int G,
                      __nv_bfloat16* __restrict__ y, __nv_bfloat16* __restrict__ yT,
                      uint32_t* __restrict__ fix_list, unsigned int* __restrict__ fix_count) {
    using Cfg = PhiGemmCfg<D>;
    constexpr int NH = Cfg::NH;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    double* acc = reinterpret_cast<double*>(smem + Cfg::kStages * Cfg::kStageBytes);   // [NH][128]
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kStages * Cfg::kStageBytes + Cfg::kAccBytes);
    uint64_t* empty = full + Cfg::kStages;
    uint64_t* cfull = empty + Cfg::kStages;   // [2]
    uint64_t* cfree = cfull + 2;              // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cfree + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int i0 = blockIdx.x * 128, g = blockIdx.y >> 1, half = blockIdx.y & 1, b = blockIdx.z;
    const int nk = l * (D / 64);
    const int nchunks = (nk + kPhiChunk - 1) / kPhiChunk;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&cfull[s], 1);
            mbar_init(&cfree[s], 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0) {
            tma_prefetch_desc(&mapA);
            tma_prefetch_desc(&mapW);
            for (int ks = 0; ks < nk; ++ks) {
                const int s = ks % Cfg::kStages;
                if (ks >= Cfg::kStages &&
                    !wait_or_abort(&empty[s], ((ks / Cfg::kStages) - 1) & 1, 0x101, abort_flag))
                    break;
                const int j = ks / (D / 64), cc = ks % (D / 64);
                uint8_t* sa = smem + s * Cfg::kStageBytes;
                uint8_t* sb = sa + Cfg::kABytes;
                mbar_expect_tx(&full[s], Cfg::kStageBytes);
                tma_load_5d(sa, &mapA, &full[s], cc * 64, g, j % d, i0 + j / d, b);
                tma_load_2d(sb, &mapW, &full[s], j * D + cc * 64, half * NH);
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(128, NH);
            bool ok = true;
            for (int ch = 0; ch < nchunks && ok; ++ch) {
                const int buf = ch & 1;
                if (ch >= 2 && !wait_or_abort(&cfree[buf], ((ch - 2) >> 1) & 1, 0x104, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kc = 0; kc < kPhiChunk && ch * kPhiChunk + kc < nk; ++kc) {
                    const int ks = ch * kPhiChunk + kc;
                    const int s = ks % Cfg::kStages;
                    if (!wait_or_abort(&full[s], (ks / Cfg::kStages) & 1, 0x102, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * Cfg::kStageBytes);
                    const uint32_t sb = sa + Cfg::kABytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16_ss(tmem + buf * NH, sdesc_sw128(sa + kk * 32), sdesc_sw128(sb + kk * 32),
                                     idesc, (kc > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[s]);
                }
                umma_commit(&cfull[buf]);
            }
        }
    } else {
        // epilogue: thread = row (compressed block i0 + row); fp64 accumulation
        const int row = threadIdx.x;
        const uint32_t tbase = tmem + ((uint32_t)(warp * 32) << 16);
        bool ok = true;
        for (int ch = 0; ch < nchunks; ++ch) {
            const int buf = ch & 1;
            if (ok) ok = wait_or_abort(&cfull[buf], (ch >> 1) & 1, 0x103, abort_flag);
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < NH; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(tbase + buf * NH + c0, r);
                tmem_wait_ld32(r);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    double* a = acc + (size_t)(c0 + e) * 128 + row;
                    *a = (ch == 0 ? 0.0 : *a) + (double)__uint_as_float(r[e]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&cfree[buf]);
        }
        const int i = i0 + row;
        if (ok && !*abort_flag && i < C) {
            for (int c = 0; c < NH; ++c) {
                const int o = half * NH + c;
                const double v = acc[(size_t)c * 128 + row] + bias[o];
                const __nv_bfloat16 r = d2bf16_rn(v);
                if (y) y[(((size_t)blockIdx.z * C + i) * G + g) * D + o] = r;
                if (yT) yT[(((size_t)blockIdx.z * G + g) * D + o) * Cp + i] = r;
                if (near_bf16_midpoint(v)) {
                    const unsigned slot = atomicAdd(fix_count, 1u);
                    fix_list[slot] = (uint32_t)((((size_t)blockIdx.z * C + i) * G + g) * D + o);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::kTmemCols);
    }
}

// Exact recomputation of the listed elements: one warp per element, the fp64
// bias W[o,:]·E (computed once by phi_bias_kernel) plus the fp64 sum of
// W[o, x] * x_blk[x] over the l*D inputs (8 per lane and load); each bf16
// product is exact in fp32, so one widening per product remains.  Rounded once.
template <int D>
__global__ void __launch_bounds__(256)
    phi_fixup_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ W,
                     const double* __restrict__ bias, int T, int G, int l, int d, int C, int Cp,
                     const uint32_t* __restrict__ fix_list, const unsigned int* __restrict__ fix_count,
                     __nv_bfloat16* __restrict__ y, __nv_bfloat16* __restrict__ yT) {
    const int lane = threadIdx.x & 31;
    const unsigned n = *fix_count;
    const unsigned nwarps = gridDim.x * (blockDim.x / 32);
    for (unsigned w = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; w < n; w += nwarps) {
        const uint32_t e = fix_list[w];
        const int o = e % D;
        uint32_t rest = e / D;
        const int g = rest % G;
        rest /= G;
        const int i = rest % C;
        const int b = rest / C;
        double acc0 = 0.0, acc1 = 0.0;
        const __nv_bfloat16* wr = W + (size_t)o * l * D;
        // unrolled so that eight iterations' loads are in flight together (the
        // summation order is unchanged)
#pragma unroll 8
        for (int xx = lane * 8; xx < l * D; xx += 256) {
            const int j = xx / D, c = xx % D;
            const uint4 xv = *reinterpret_cast<const uint4*>(
                x + (((size_t)b * T + (size_t)i * d + j) * G + g) * D + c);
            const uint4 wv = *reinterpret_cast<const uint4*>(wr + xx);
            const __nv_bfloat16* xh = reinterpret_cast<const __nv_bfloat16*>(&xv);
            const __nv_bfloat16* wh = reinterpret_cast<const __nv_bfloat16*>(&wv);
#pragma unroll
            for (int q = 0; q < 8; q += 2) {
                acc0 += (double)(__bfloat162float(wh[q]) * __bfloat162float(xh[q]));
                acc1 += (double)(__bfloat162float(wh[q + 1]) * __bfloat162float(xh[q + 1]));
            }
        }
        double acc = acc0 + acc1;
#pragma unroll
        for (int s2 = 16; s2 >= 1; s2 >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s2);
        if (lane == 0) {
            const __nv_bfloat16 r = d2bf16_rn(acc + bias[o]);
            if (y) y[(((size_t)b * C + i) * G + g) * D + o] = r;
            if (yT) yT[(((size_t)b * G + g) * D + o) * Cp + i] = r;
        }
    }
}

// ------------------------------------------------------------- v transpose
// v [B,T,G,D] -> vT [B,G,DP,Tp] (Tp = T rounded up to 8, DP >= D rows, rows
// D..DP-1 and columns T..Tp-1 zero): the K-major operand layout of the P.V
// products.  grid (ceil(Tp/64), G, B), block (64, 4).
__global__ void transpose_v_kernel(const __nv_bfloat16* __restrict__ v, int T, int G, int D, int DP,
                                   int Tp, __nv_bfloat16* __restrict__ vT) {
    __shared__ __nv_bfloat16 tile[64][65];
    const int t0 = blockIdx.x * 64, g = blockIdx.y, b = blockIdx.z;
    for (int c0 = 0; c0 < DP; c0 += 64) {
        for (int tt = threadIdx.y; tt < 64; tt += blockDim.y) {
            const int t = t0 + tt, c = c0 + threadIdx.x;
            tile[tt][threadIdx.x] = (t < T && c < D) ? v[(((size_t)b * T + t) * G + g) * D + c]
                                                     : __float2bfloat16_rn(0.f);
        }
        __syncthreads();
        for (int cc = threadIdx.y; cc < 64; cc += blockDim.y) {
            const int c = c0 + cc, t = t0 + threadIdx.x;
            if (c < DP && t < Tp) vT[(((size_t)b * G + g) * DP + c) * Tp + t] = tile[threadIdx.x][cc];
        }
        __syncthreads();
    }
}

}  // namespace nsa
