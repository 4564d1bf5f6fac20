// k_backward.cuh -- backward of the NSA operator with the block selection held
// fixed (pages: natively trainable design, 效率分析 training speed).
//
// Per branch c with dO_c = g_c dO (softmax backward):
//   P = exp(S - LSE_c), dP_u = <dO_c, V_u>, D_c = <dO_c, o_c>,
//   dS = P (dP - D_c), dq += scale dS K, dK_u += scale dS q, dV_u += P dO_c,
//   d(gate_c) = <dO, o_c>.
// The compressed branch's dK~/dV~ go back through phi (mean: /l to each
// member token; linear: W^T dK~ scattered over the overlapping blocks).
//
// Kernels of this file (the tcgen05 passes live in k_bwd_kv.cuh: key-centric
// dK/dV; k_bwd_q.cuh: dq of the window and compressed branches; k_bwd_qsel.cuh:
// dq of the selected branch):
//   bwd_branch_stats     d(gate_c), D_c and the log2 LSE of one branch from its
//                        output under unit gates (the forward's kernels).
//   bwd_phiT_kernel      dk/dv += phi^T(dK~/dV~).
#pragma once
#include "nsa_dev.cuh"

namespace nsa {

enum { kBrCmp = 0, kBrSlc = 1, kBrWin = 2 };

struct BwdParams {
    int B, T, H, G, HG, DK, DV, l, d, lp, n, w, C, NSb;
    float scale, scale_log2;
    const __nv_bfloat16 *q, *k, *v, *kc, *vc, *dout, *wk, *wv;
    const float* gates;
    const int32_t* idx;
    float *dq, *dk, *dv, *dgates;
    float *lse2, *dlt;          // [B,T,H,3]
    float *dkc, *dvc;           // [B,C,G,*]
    int *cnt, *cursor, *off, *chunk_off, *list;
    int phi;                    // 0 mean, 1 linear
};

__device__ __forceinline__ int ncmp_vis(const BwdParams& p, int t) {
    return (t + 1 >= p.l) ? (t + 1 - p.l) / p.d + 1 : 0;
}

// ------------------------------------------------- per-branch statistics
// From one branch's output o_c (computed with unit gates) and its natural-log
// LSE: d(gate_c) = <dO, o_c>, D_c = g_c <dO, o_c>, LSE in log2 units.  One
// warp per query row (b, t, h).
__global__ void bwd_branch_stats(const float* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                                 const float* __restrict__ gates, const float* __restrict__ lse_nat, int br,
                                 long long rows, int DV, float* dgates, float* dlt, float* lse2) {
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float acc = 0.f;
    for (int c = lane * 4; c < DV; c += 128) {
        const float4 ov = *reinterpret_cast<const float4*>(o + row * DV + c);
        const uint2 dv = *reinterpret_cast<const uint2*>(dout + row * DV + c);
        const __nv_bfloat162 d01 = *reinterpret_cast<const __nv_bfloat162*>(&dv.x);
        const __nv_bfloat162 d23 = *reinterpret_cast<const __nv_bfloat162*>(&dv.y);
        acc += ov.x * __low2float(d01) + ov.y * __high2float(d01) + ov.z * __low2float(d23) +
               ov.w * __high2float(d23);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (lane == 0) {
        dgates[row * 3 + br] = acc;
        dlt[row * 3 + br] = gates[row * 3 + br] * acc;
        lse2[row * 3 + br] = lse_nat[row * 3 + br] * kLog2e;
    }
}

// All three branches at once from their saved outputs o_c [3][rows][DV] (the
// training forward's): dO is read once per row instead of once per branch.
__global__ void bwd_branch_stats3(const float* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                                  const float* __restrict__ gates, const float* __restrict__ lse_nat, long long rows,
                                  int DV, float* dgates, float* dlt, float* lse2) {
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float acc[3] = {0.f, 0.f, 0.f};
    for (int c = lane * 4; c < DV; c += 128) {
        const uint2 dv = *reinterpret_cast<const uint2*>(dout + row * DV + c);
        const __nv_bfloat162 d01 = *reinterpret_cast<const __nv_bfloat162*>(&dv.x);
        const __nv_bfloat162 d23 = *reinterpret_cast<const __nv_bfloat162*>(&dv.y);
#pragma unroll
        for (int br = 0; br < 3; ++br) {
            const float4 ov = *reinterpret_cast<const float4*>(o + ((size_t)br * rows + row) * DV + c);
            acc[br] += ov.x * __low2float(d01) + ov.y * __high2float(d01) + ov.z * __low2float(d23) +
                       ov.w * __high2float(d23);
        }
    }
#pragma unroll
    for (int br = 0; br < 3; ++br)
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) acc[br] += __shfl_xor_sync(0xffffffffu, acc[br], m);
    if (lane < 3) {
        const int br = lane;
        const float a = br == 0 ? acc[0] : br == 1 ? acc[1] : acc[2];
        dgates[row * 3 + br] = a;
        dlt[row * 3 + br] = gates[row * 3 + br] * a;
        lse2[row * 3 + br] = lse_nat[row * 3 + br] * kLog2e;
    }
}

__global__ void fill_f32(float* x, long long n, float v) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) x[i] = v;
}

// ------------------------------------------------------------ phi^T
// dX[b,u,g,c] += sum over blocks i containing u of (W^T dY[b,i,g])[ (u - i*d)*D + c ]
// (mean: dY[b,i,g,c] / l).  grid (T, G, B), block D.
template <int D>
__global__ void bwd_phiT_kernel(const BwdParams p, const float* __restrict__ dY,
                                const __nv_bfloat16* __restrict__ W, float* __restrict__ dX) {
    __shared__ float dy[4][D];
    const int u = blockIdx.x, g = blockIdx.y, b = blockIdx.z, c = threadIdx.x;
    const int ilo = max(0, (u - p.l + p.d) / p.d), ihi = min(p.C - 1, u / p.d);
    float acc = 0.f;
    int slot = 0;
    for (int i = ilo; i <= ihi; ++i, ++slot) {
        if (u < i * p.d || u >= i * p.d + p.l) continue;
        const int j = u - i * p.d;
        const float* src = dY + (((size_t)b * p.C + i) * p.G + g) * D;
        if (p.phi == 0) {
            acc += src[c] / (float)p.l;
        } else {
            __syncthreads();
            dy[0][c] = src[c];
            __syncthreads();
            for (int o = 0; o < D; ++o)
                acc += __bfloat162float(W[(size_t)o * (p.l * D) + j * D + c]) * dy[0][o];
        }
    }
    dX[(((size_t)b * p.T + u) * p.G + g) * D + c] += acc;
}

}  // namespace nsa
