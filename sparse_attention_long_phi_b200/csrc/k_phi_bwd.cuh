// k_phi_bwd.cuh -- the linear compression map's backward products on tcgen05
// tensor cores (page "硬件对齐+原生训练！DeepSeek NSA打造高效稀疏Attention",
// 令牌压缩: K~[i] = W vec(k_blk(i) + E), block i covering tokens i*d .. i*d + l - 1,
// vec position-major: x = j*D + c).  From the compressed-key gradient
// dY = dK~ [B, C, G, D] (rounded to bf16 for the products, fp32 accumulate):
//
//   kPhiT:  dX[b, i*d + j, g, c] += sum_o dY[b,i,g,o] W[o, j*D + c]
//           M = 128 blocks i, N = 256 inputs x, K = the D outputs o;
//           A = dY (K-major), B = W (MN-major: x is contiguous).
//           Each token lies in l/d blocks, so the epilogue adds into dX.
//   kPhiDW: dW[o, x] = sum_(b,g,i) dY[b,i,g,o] vec(k_blk)[x] + s[o] E[x],
//           s[o] = sum_n dY[n, o] (given), the position embedding's share;
//           M = 128 outputs o, N = 256 inputs x, K = every (b, g, i);
//           A = dY^T (MN-major), B = the token rows of k through a 5-D view
//           {D, G, d, T/d, B} (MN-major), 64 blocks per K chunk.
//
// One CTA per output tile.  Warp 4 loads through a ring of 48 KB stages, warp
// 5 issues the MMAs into one 256-column TMEM accumulator, warps 0-3 (one TMEM
// lane quadrant each, thread = tile row) run the epilogue.
#pragma once
#include "nsa_dev.cuh"
#include "k_attn_packed.cuh"   // wait_or_abort
#include "k_bwd_kv.cuh"        // sdesc_sw128_mn, red_add_v4

namespace nsa {

enum { kPhiT = 0, kPhiDW = 1 };

struct PhiBwdCfg {
    static constexpr int NT = 256;                   // tile columns (inputs x)
    static constexpr int kABytes = 128 * 128;        // 128 rows x 64 bf16
    static constexpr int kBBytes = 4 * 64 * 128;     // 4 boxes of 64 K-rows x 64 bf16
    static constexpr int kStage = kABytes + kBBytes;
    static constexpr int kStages = 4;
    static constexpr int kSmem = kStages * kStage + 256 + 1024;
    static constexpr int kThreads = 192;
};

struct PhiBwdParams {
    int B, T, G, C, D, l, d;
    float* dX;               // kPhiT: [B, T, G, D] token gradients (added into)
    float* dW;               // kPhiDW: [D, l*D]
    const float* s;          // kPhiDW: [D] column sums of dY
    const __nv_bfloat16* E;  // kPhiDW: [l, D] position embedding
};

template <int MODE>
__global__ void __launch_bounds__(192, 1)
    phi_bwd_gemm(const __grid_constant__ CUtensorMap mapY, const __grid_constant__ CUtensorMap mapB,
                 const PhiBwdParams p) {
    using Cfg = PhiBwdCfg;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kStages * Cfg::kStage);
    uint64_t* empty = full + Cfg::kStages;
    uint64_t* accfull = empty + Cfg::kStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfull + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int x0 = blockIdx.x * Cfg::NT;     // first input column x of the tile
    const int m0 = blockIdx.y * 128;         // first block i (kPhiT) or output o (kPhiDW)
    const int bg = blockIdx.z;               // kPhiT: (b, g)
    const int nci = (p.C + 63) / 64;         // kPhiDW: K chunks of 64 blocks per (b, g)
    const int nk = MODE == kPhiT ? p.D / 64 : p.B * p.G * nci;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accfull, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&mapY);
            tma_prefetch_desc(&mapB);
            for (int kc = 0; kc < nk; ++kc) {
                const int s = kc % Cfg::kStages;
                if (kc >= Cfg::kStages &&
                    !wait_or_abort(&empty[s], ((kc / Cfg::kStages) - 1) & 1, 0x701, abort_flag))
                    break;
                uint8_t* sa = smem + s * Cfg::kStage;
                uint8_t* sb = sa + Cfg::kABytes;
                mbar_expect_tx(&full[s], Cfg::kStage);
                if (MODE == kPhiT) {
                    const int b = bg / p.G, g = bg % p.G;
                    // A: 128 blocks x 64 outputs; B: 64 outputs x 4 x 64 inputs
                    tma_load_4d(sa, &mapY, &full[s], kc * 64, g, m0, b);
#pragma unroll
                    for (int q = 0; q < 4; ++q) tma_load_2d(sb + q * 8192, &mapB, &full[s], x0 + q * 64, kc * 64);
                } else {
                    const int pair = kc / nci, i0 = (kc % nci) * 64;
                    const int b = pair / p.G, g = pair % p.G;
                    // A: 64 blocks x 2 x 64 outputs; B: 64 blocks x 4 x 64 inputs (one
                    // position j per 64 inputs: token row i*d + j of block i)
#pragma unroll
                    for (int h = 0; h < 2; ++h) tma_load_4d(sa + h * 8192, &mapY, &full[s], m0 + h * 64, g, i0, b);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int x = x0 + q * 64, j = x / p.D, c0 = x - j * p.D;
                        tma_load_5d(sb + q * 8192, &mapB, &full[s], c0, g, j % p.d, i0 + j / p.d, b);
                    }
                }
            }
        }
    } else if (warp == 5) {
        // ----------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idesc =
                idesc_bf16(128, Cfg::NT) | (1u << 16) | (MODE == kPhiDW ? (1u << 15) : 0u);
            bool ok = true;
            for (int kc = 0; kc < nk && ok; ++kc) {
                const int s = kc % Cfg::kStages;
                if (!(ok = wait_or_abort(&full[s], (kc / Cfg::kStages) & 1, 0x702, abort_flag))) break;
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + s * Cfg::kStage);
                const uint32_t sb = sa + Cfg::kABytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t da = MODE == kPhiT ? sdesc_sw128(sa + kk * 32) : sdesc_sw128_mn(sa + kk * 2048, 8192, 1024);
                    umma_bf16_ss(tmem, da, sdesc_sw128_mn(sb + kk * 2048, 8192, 1024), idesc,
                                 (kc > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&empty[s]);
            }
            umma_commit(accfull);
        }
    } else {
        // ------------------------------------------------------ epilogue
        const int row = m0 + warp * 32 + lane;
        const uint32_t tbase = tmem + ((uint32_t)(warp * 32) << 16);
        bool ok = true;
        if (lane == 0) ok = wait_or_abort(accfull, 0, 0x703, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        tc_fence_after();
        const bool live = ok && (MODE == kPhiT ? row < p.C : row < p.D);
        const int b = bg / p.G, g = bg % p.G;
        const float srow = (MODE == kPhiDW && live) ? p.s[row] : 0.f;
#pragma unroll 1
        for (int c0 = 0; c0 < Cfg::NT; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(tbase + c0, r);
            tmem_wait_ld32(r);
            if (!live) continue;
            // 32 columns lie inside one position j (D is a multiple of 64)
            const int x = x0 + c0, j = x / p.D, c = x - j * p.D;
            if (MODE == kPhiT) {
                const int u = row * p.d + j;       // token of position j in block `row`
                if (u < p.T) {
                    float* dst = p.dX + (((size_t)b * p.T + u) * p.G + g) * p.D + c;
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        red_add_v4(dst + e, __uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                                   __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
                }
            } else {
                float4* dst = reinterpret_cast<float4*>(p.dW + (size_t)row * p.l * p.D + x);
                const __nv_bfloat16* e = p.E + (size_t)j * p.D + c;
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    dst[q] = make_float4(
                        fmaf(srow, __bfloat162float(e[4 * q + 0]), __uint_as_float(r[4 * q + 0])),
                        fmaf(srow, __bfloat162float(e[4 * q + 1]), __uint_as_float(r[4 * q + 1])),
                        fmaf(srow, __bfloat162float(e[4 * q + 2]), __uint_as_float(r[4 * q + 2])),
                        fmaf(srow, __bfloat162float(e[4 * q + 3]), __uint_as_float(r[4 * q + 3])));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// fp32 -> bf16 (round to nearest even), n a multiple of 4
__global__ void f32_to_bf16_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y, long long n4) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    const float4 v = reinterpret_cast<const float4*>(x)[i];
    uint2 o;
    o.x = pack_bf16x2(v.x, v.y);
    o.y = pack_bf16x2(v.z, v.w);
    reinterpret_cast<uint2*>(y)[i] = o;
}

}  // namespace nsa
