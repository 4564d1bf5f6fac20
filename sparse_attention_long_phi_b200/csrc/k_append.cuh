// k_append.cuh -- decode-step cache maintenance (page "硬件对齐+原生训练！DeepSeek
// NSA打造高效稀疏Attention", 令牌压缩 and 效率分析 解码速度): the decode step reads a
// raw K/V cache and a compressed K~/V~ cache; each generated token is appended to
// the raw cache, and every d tokens (once at least l are present) a compressed
// block i = (L - l)/d completes and its phi is appended to the compressed cache.
//
// kAppendSplit CTAs per (sequence, group, K or V), each owning a slice of the
// outputs; the first copies the new token's row into the raw cache.  If that
// token completes a block, each CTA stages the block's x = vec(k_blk + E) in
// fp64 in shared memory and computes its outputs: each one fp64 dot product
// (linear: W[o,:] . x; mean: the average of the l rows), rounded once to bf16
// (round to nearest even), so the result is the correctly rounded phi with no
// fix-up pass.  The block's last row is the new token itself, read from the
// input rather than from the cache, so the copy and the compression need no
// ordering.
#pragma once
#include "nsa_dev.cuh"
#include "k_phi.cuh"   // d2bf16_rn

namespace nsa {

struct AppendParams {
    int S, G, l, d, phi;           // phi: 0 mean, 1 linear
    const int64_t* kv_start;       // [S] row of token 0 of sequence s in the raw caches
    const int64_t* cmp_start;      // [S] row of compressed block 0 of sequence s
    const int64_t* len;            // [S] tokens already cached (the new token's position)
    const __nv_bfloat16 *k_new, *v_new;   // [S,G,D]
    __nv_bfloat16 *k_cache, *v_cache;     // [rows,G,D]
    __nv_bfloat16 *kc_cache, *vc_cache;   // [rows,G,D]
    const __nv_bfloat16 *w_k, *e_k, *w_v, *e_v;   // linear phi: W [D, l*D], E [l, D]
};

constexpr int kAppendSplit = 8;   // CTAs per (sequence, group, K or V): output slices

template <int D>
__device__ __forceinline__ void append_one(const AppendParams& p, int s, int g, int isv, int part, double* xs) {
    const int64_t L0 = p.len[s];                      // position of the new token
    const __nv_bfloat16* xn = (isv ? p.v_new : p.k_new) + ((size_t)s * p.G + g) * D;
    __nv_bfloat16* cache = isv ? p.v_cache : p.k_cache;
    const __nv_bfloat16* crow = cache + (size_t)p.kv_start[s] * p.G * D + g * D;   // token 0, group g
    // 1. the new token's row (slice 0)
    if (part == 0)
        for (int c = threadIdx.x; c < D / 8; c += blockDim.x)
            reinterpret_cast<uint4*>(cache + ((size_t)(p.kv_start[s] + L0) * p.G + g) * D)[c] =
                reinterpret_cast<const uint4*>(xn)[c];
    // 2. the compressed block it completes, if any
    const int64_t L1 = L0 + 1;
    if (L1 < p.l || (L1 - p.l) % p.d != 0) return;
    const int64_t i = (L1 - p.l) / p.d;              // block i covers tokens [i*d, i*d + l)
    const int64_t t0 = i * p.d;
    __nv_bfloat16* dst = (isv ? p.vc_cache : p.kc_cache) + ((size_t)(p.cmp_start[s] + i) * p.G + g) * D;
    // row j of the block (token t0 + j): the input for the new token, else the cache
    auto row = [&](int j) -> const __nv_bfloat16* {
        return (t0 + j == L0) ? xn : crow + (size_t)(t0 + j) * p.G * D;
    };
    constexpr int OPC = D / kAppendSplit;            // outputs of this CTA: [part*OPC, part*OPC + OPC)
    if (p.phi == 0) {
        for (int c = part * OPC + threadIdx.x; c < part * OPC + OPC; c += blockDim.x) {
            double acc = 0.0;
#pragma unroll 8
            for (int j = 0; j < p.l; ++j) acc += (double)__bfloat162float(row(j)[c]);
            dst[c] = d2bf16_rn(acc / (double)p.l);
        }
        return;
    }
    // linear: x = vec(k_blk + E) staged once in fp64 (exact sums of two bf16
    // values), 8 elements (one 16-byte load of the row and of E) per step
    const __nv_bfloat16* W = isv ? p.w_v : p.w_k;
    const __nv_bfloat16* E = isv ? p.e_v : p.e_k;
    const int K = p.l * D;                            // position-major: x[j*D + c]
#pragma unroll 4
    for (int x8 = threadIdx.x; x8 < K / 8; x8 += blockDim.x) {
        const int j = (x8 * 8) / D, c = x8 * 8 - j * D;
        const uint4 kv = *reinterpret_cast<const uint4*>(row(j) + c);
        const uint4 ev = reinterpret_cast<const uint4*>(E)[x8];
        const __nv_bfloat16* kh = reinterpret_cast<const __nv_bfloat16*>(&kv);
        const __nv_bfloat16* eh = reinterpret_cast<const __nv_bfloat16*>(&ev);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            xs[x8 * 8 + e] = (double)__bfloat162float(kh[e]) + (double)__bfloat162float(eh[e]);
    }
    __syncthreads();
    // each warp: OPW outputs at once (independent accumulators, loads in flight together)
    constexpr int OPW = OPC / 8;                      // 8 warps
    static_assert(OPW >= 1 && OPC % 8 == 0, "outputs per warp");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int o0 = part * OPC + warp * OPW;
    double acc[OPW];
#pragma unroll
    for (int u = 0; u < OPW; ++u) acc[u] = 0.0;
#pragma unroll 2
    for (int x8 = lane; x8 < K / 8; x8 += 32) {
        uint4 wv[OPW];
#pragma unroll
        for (int u = 0; u < OPW; ++u) wv[u] = reinterpret_cast<const uint4*>(W + (size_t)(o0 + u) * K)[x8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const double xv = xs[x8 * 8 + e];
#pragma unroll
            for (int u = 0; u < OPW; ++u)
                acc[u] = fma((double)__bfloat162float(reinterpret_cast<const __nv_bfloat16*>(&wv[u])[e]), xv, acc[u]);
        }
    }
#pragma unroll
    for (int u = 0; u < OPW; ++u) {
        double a = acc[u];
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) a += __shfl_xor_sync(0xffffffffu, a, m);
        if (lane == 0) dst[o0 + u] = d2bf16_rn(a);
    }
}

// grid (S, G, 2 * kAppendSplit), block 256, dynamic shared memory l * max(DK, DV)
// doubles: z / kAppendSplit = 0 for K (width DK), 1 for V (width DV); z % kAppendSplit
// = the slice of the outputs this CTA computes.
template <int DK, int DV>
__global__ void __launch_bounds__(256) decode_append_kernel(const AppendParams p) {
    extern __shared__ double xs[];
    const int isv = blockIdx.z / kAppendSplit, part = blockIdx.z % kAppendSplit;
    if (isv) append_one<DV>(p, blockIdx.x, blockIdx.y, 1, part, xs);
    else append_one<DK>(p, blockIdx.x, blockIdx.y, 0, part, xs);
}

}  // namespace nsa
