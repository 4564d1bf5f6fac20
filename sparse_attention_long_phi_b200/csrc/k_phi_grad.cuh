// k_phi_grad.cuh -- gradients of the linear compression map's parameters (page
// "硬件对齐+原生训练！DeepSeek NSA打造高效稀疏Attention", 令牌压缩: the compression is a
// learnable map with an intra-block position encoding, K~[i] = W vec(k_blk + E)).
// From the compressed-key gradients dY = dK~ [N = B*C*G, D] of the backward:
//   dW[o, x]  = sum_n dY[n, o] * X[n, x],   X[n] = vec(k_blk(n) + E)   [D, l*D]
//   dE[j, c]  = sum_o W[o, j*D + c] * s[o], s[o] = sum_n dY[n, o]       [l, D]
// fp32 throughout (the gradients' tolerance is a relative L2 of 1e-2); the bf16
// rounding of K~ is treated as the identity, as in the rest of the backward.
#pragma once
#include "nsa_dev.cuh"

namespace nsa {

// dW tile [64 outputs o] x [64 inputs x] per CTA, summed over n in chunks of 32
// rows staged in shared memory; X rebuilt from the token rows (k + E) on load.
// grid (l*D/64, D/64), block 256 (thread: 4 x 4 outputs).  D % 64 == 0, so a
// 64-wide x tile lies inside one block position j.
template <int D>
__global__ void __launch_bounds__(256) phi_dw_kernel(const float* __restrict__ dY, const __nv_bfloat16* __restrict__ x,
                                                     const __nv_bfloat16* __restrict__ E, int B, int T, int G, int C,
                                                     int l, int d, float* __restrict__ dW) {
    __shared__ __align__(16) float sA[32][64];   // dY rows x outputs
    __shared__ __align__(16) float sB[32][64];   // X rows x inputs
    const int x0 = blockIdx.x * 64, o0 = blockIdx.y * 64;
    const int j = x0 / D, c0 = x0 - j * D;
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int N = B * C * G;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b2 = 0; b2 < 4; ++b2) acc[a][b2] = 0.f;
    for (int n0 = 0; n0 < N; n0 += 32) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int e = tid + k * 256, r = e >> 6, cc = e & 63, n = n0 + r;
            float av = 0.f, bv = 0.f;
            if (n < N) {
                const int g = n % G, bi = n / G, i = bi % C, b = bi / C;
                av = dY[(size_t)n * D + o0 + cc];
                bv = __bfloat162float(x[(((size_t)b * T + (size_t)i * d + j) * G + g) * D + c0 + cc]) +
                     __bfloat162float(E[j * D + c0 + cc]);
            }
            sA[r][cc] = av;
            sB[r][cc] = bv;
        }
        __syncthreads();
#pragma unroll 8
        for (int r = 0; r < 32; ++r) {
            const float4 a4 = *reinterpret_cast<const float4*>(&sA[r][ty * 4]);
            const float4 b4 = *reinterpret_cast<const float4*>(&sB[r][tx * 4]);
            const float av[4] = {a4.x, a4.y, a4.z, a4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b2 = 0; b2 < 4; ++b2) acc[a][b2] = fmaf(av[a], bv[b2], acc[a][b2]);
        }
        __syncthreads();
    }
    const int K = l * D;
#pragma unroll
    for (int a = 0; a < 4; ++a)
        *reinterpret_cast<float4*>(dW + (size_t)(o0 + ty * 4 + a) * K + x0 + tx * 4) =
            make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
}

// s[o] = sum_n dY[n, o] in two steps.  phi_colsum_kernel: grid (D/32, NB), block
// 256 (lane = column); CTA y takes rows n = y, y + NB, ..., warp w of them every
// eighth, and writes its sum to part[y][o] (the eight warps added in a fixed
// order).  phi_colsum_fold: s[o] = part[0][o] + ... + part[NB-1][o] in order.
__global__ void __launch_bounds__(256) phi_colsum_kernel(const float* __restrict__ dY, int N, int D, int NB,
                                                         float* __restrict__ part) {
    __shared__ float red[8][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, o = blockIdx.x * 32 + lane;
    float acc = 0.f;
#pragma unroll 8
    for (int n = blockIdx.y + NB * warp; n < N; n += NB * 8) acc += dY[(size_t)n * D + o];
    red[warp][lane] = acc;
    __syncthreads();
    if (warp == 0) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) t += red[w][lane];
        part[(size_t)blockIdx.y * D + o] = t;
    }
}

__global__ void phi_colsum_fold(const float* __restrict__ part, int NB, int D, float* __restrict__ s) {
    const int o = blockIdx.x * blockDim.x + threadIdx.x;
    if (o >= D) return;
    float t = 0.f;
    for (int y = 0; y < NB; ++y) t += part[(size_t)y * D + o];
    s[o] = t;
}

// dE[x] = sum_o W[o, x] s[o]: one thread per x of the l*D inputs.
__global__ void __launch_bounds__(256) phi_de_kernel(const __nv_bfloat16* __restrict__ W, const float* __restrict__ s,
                                                     int D, int K, float* __restrict__ dE) {
    const int xx = blockIdx.x * blockDim.x + threadIdx.x;
    if (xx >= K) return;
    float acc = 0.f;
#pragma unroll 4
    for (int o = 0; o < D; ++o) acc = fmaf(__bfloat162float(W[(size_t)o * K + xx]), s[o], acc);
    dE[xx] = acc;
}

}  // namespace nsa
