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
// Kernels of this file (the tcgen05 key-centric and dense query-centric
// passes live in k_bwd_kv.cuh and k_bwd_q.cuh):
//   bwd_query_mma        one CTA per (b, t, g) on warp-level bf16 tensor cores
//                        (the 16 heads of the group are the M side): with the
//                        row statistics known, recomputes S and dP = dO_c V^T
//                        over the selected blocks, forms dS and accumulates
//                        dq = scale dS K (sweep 2); without them it first
//                        recomputes every branch's LSE and o_c (sweep 1).
//   bwd_branch_stats     d(gate_c), D_c and the log2 LSE of one branch from its
//                        output under unit gates.
//   bwd_phiT_kernel      dk/dv += phi^T(dK~/dV~).
#pragma once
#include "nsa_dev.cuh"
#include "k_mma.cuh"

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
    int have_stats;             // lse2 / dlt / dgates already computed: the query pass skips its sweep 1
    int q_branches;             // bit br set: the query pass accumulates dq of branch br (sweep 2)
};

__device__ __forceinline__ int ncmp_vis(const BwdParams& p, int t) {
    return (t + 1 >= p.l) ? (t + 1 - p.l) / p.d + 1 : 0;
}

// ------------------------------------------------ per query, tensor cores
// Shared memory: 4 warps x (32 K rows + 32 V rows) staging (reused for the
// cross-warp merges), then dO_t of the group as a [16][DV] bf16 tile.
template <int DK, int DV>
constexpr int bwd_query_mma_smem() {
    return 4 * 32 * ((DK * 2 + 16) + (DV * 2 + 16)) + 16 * (DV * 2 + 16);
}

template <int DK, int DV>
__global__ void __launch_bounds__(128) bwd_query_mma(const BwdParams p) {
    constexpr int KP = DK * 2 + 16, VP = DV * 2 + 16;
    constexpr int STAGE = 4 * 32 * (KP + VP);
    static_assert(4 * 16 * DK * 4 <= STAGE && 4 * 16 * DV * 4 <= STAGE, "merge buffers");
    extern __shared__ __align__(16) uint8_t bsm[];
    __shared__ float wm[4][16], wl[4][16], Lsum[16];
    __shared__ float lse2s[3][16], Ds[3][16], gs[3][16];
    __shared__ int units[16];
    __shared__ int nunits;
    const int t = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gr = lane >> 2, tg = lane & 3;
    const size_t rowbase = ((size_t)b * p.T + t) * p.H + (size_t)g * p.HG;
    uint8_t* ks = bsm + warp * 32 * (KP + VP);
    uint8_t* vs = ks + 32 * KP;
    uint8_t* dos = bsm + STAGE;
    if (threadIdx.x == 0) {
        int nu = 0;
        const int32_t* r = p.idx + (((size_t)b * p.T + t) * p.G + g) * p.n;
        for (int a = 0; a < p.n; ++a)
            if (r[a] >= 0) units[nu++] = r[a];
        nunits = nu;
    }
    for (int e = threadIdx.x; e < 16 * (DV / 8); e += 128) {     // dO tile, zero rows past HG
        const int h = e / (DV / 8), cc = e % (DV / 8);
        int4 v = make_int4(0, 0, 0, 0);
        if (h < p.HG) v = *reinterpret_cast<const int4*>(p.dout + (rowbase + h) * DV + cc * 8);
        *reinterpret_cast<int4*>(dos + h * VP + cc * 16) = v;
    }
    if (threadIdx.x < 48) {
        const int br = threadIdx.x / 16, h = threadIdx.x % 16;
        gs[br][h] = h < p.HG ? p.gates[(rowbase + h) * 3 + br] : 0.f;
    }
    __syncthreads();
    uint32_t qa[DK / 16][4];
    load_a_frags<DK>(p.q + rowbase * DK, p.HG, qa);
    const float c = p.scale_log2;

    // key range of a branch; row pointers (nullptr: not seen by the query)
    auto branch_keys = [&](int br, int& lo) -> int {
        lo = 0;
        if (br == kBrCmp) return ncmp_vis(p, t);
        if (br == kBrSlc) return nunits * p.lp;
        lo = max(0, t - p.w + 1);
        return t - lo + 1;
    };
    // Stage the 32 keys k0.. of a branch (K rows at ks, V rows at vs) and return
    // how many of them the query sees: they are a prefix, because a chunk's rows
    // are consecutive cache rows (a selected block holds whole 32-key chunks) in
    // increasing token order.
    auto stage = [&](int br, int lo, int nk, int k0) -> int {
        int row0, nval = min(32, nk - k0);
        const __nv_bfloat16 *kb, *vb;
        if (br == kBrCmp) {
            row0 = k0;
            kb = p.kc + (((size_t)b * p.C + row0) * p.G + g) * DK;
            vb = p.vc + (((size_t)b * p.C + row0) * p.G + g) * DV;
        } else {
            if (br == kBrSlc) {
                const int ui = k0 / p.lp;
                row0 = units[ui] * p.lp + (k0 - ui * p.lp);
                nval = min(nval, t - row0 + 1);
            } else {
                row0 = lo + k0;
            }
            kb = p.k + (((size_t)b * p.T + row0) * p.G + g) * DK;
            vb = p.v + (((size_t)b * p.T + row0) * p.G + g) * DV;
        }
        warp_issue_32rows<DK>(ks, kb, (size_t)p.G * DK, nval);
        warp_issue_32rows<DV>(vs, vb, (size_t)p.G * DV, nval);
        cp_async_commit();
        cp_async_wait();
        __syncwarp();
        return nval;
    };

    // ---------------- pass 1, every branch: LSE, o_c, dgates, D
    if (p.have_stats) {
        if (threadIdx.x < 48) {
            const int br = threadIdx.x / 16, h = threadIdx.x % 16;
            lse2s[br][h] = h < p.HG ? p.lse2[(rowbase + h) * 3 + br] : -INFINITY;
            Ds[br][h] = h < p.HG ? p.dlt[(rowbase + h) * 3 + br] : 0.f;
        }
        __syncthreads();
    }
    for (int br = 0; br < 3 && !p.have_stats; ++br) {
        int lo;
        const int nk = branch_keys(br, lo);
        const int nch = (nk + 31) / 32;
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        float o[DV / 8][4];
#pragma unroll
        for (int nt = 0; nt < DV / 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
        for (int ch = warp; ch < nch; ch += 4) {
            const int k0 = ch * 32;
            const int nval = stage(br, lo, nk, k0);
            float sf[4][4];
            warp_logits<DK>(qa, smem_u32(ks), sf);
            float cm0 = -INFINITY, cm1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float v = nt * 8 + tg * 2 + (e & 1) < nval ? sf[nt][e] * c : -INFINITY;
                    sf[nt][e] = v;
                    if (e < 2) cm0 = fmaxf(cm0, v);
                    else cm1 = fmaxf(cm1, v);
                }
#pragma unroll
            for (int q2 = 1; q2 <= 2; q2 <<= 1) {
                cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, q2));
                cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, q2));
            }
            const float n0 = fmaxf(m0, cm0), n1 = fmaxf(m1, cm1);
            const float a0 = n0 == -INFINITY ? 1.f : exp2f(m0 - n0);
            const float a1 = n1 == -INFINITY ? 1.f : exp2f(m1 - n1);
            m0 = n0;
            m1 = n1;
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float mm = e < 2 ? m0 : m1;
                    const float pv = sf[nt][e] == -INFINITY ? 0.f : exp2f(sf[nt][e] - mm);
                    sf[nt][e] = pv;
                    if (e < 2) s0 += pv;
                    else s1 += pv;
                }
#pragma unroll
            for (int q2 = 1; q2 <= 2; q2 <<= 1) {
                s0 += __shfl_xor_sync(0xffffffffu, s0, q2);
                s1 += __shfl_xor_sync(0xffffffffu, s1, q2);
            }
            l0 = l0 * a0 + s0;
            l1 = l1 * a1 + s1;
#pragma unroll
            for (int nt = 0; nt < DV / 8; ++nt) {
                o[nt][0] *= a0;
                o[nt][1] *= a0;
                o[nt][2] *= a1;
                o[nt][3] *= a1;
            }
            warp_pv<DV>(sf, smem_u32(vs), o);
            __syncwarp();
        }
        // merge the 4 warps (fixed order): LSE and o_c per head
        if (tg == 0) {
            wm[warp][gr] = m0;
            wm[warp][gr + 8] = m1;
            wl[warp][gr] = l0;
            wl[warp][gr + 8] = l1;
        }
        __syncthreads();                                      // also: staging idle
        float* ored = reinterpret_cast<float*>(bsm);          // [4][16][DV]
        {
            const float M0 = fmaxf(fmaxf(wm[0][gr], wm[1][gr]), fmaxf(wm[2][gr], wm[3][gr]));
            const float M1 = fmaxf(fmaxf(wm[0][gr + 8], wm[1][gr + 8]), fmaxf(wm[2][gr + 8], wm[3][gr + 8]));
            const float f0 = m0 == -INFINITY ? 0.f : exp2f(m0 - M0);
            const float f1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M1);
#pragma unroll
            for (int nt = 0; nt < DV / 8; ++nt) {
                const int cc = nt * 8 + tg * 2;
                *reinterpret_cast<float2*>(ored + (warp * 16 + gr) * DV + cc) = make_float2(o[nt][0] * f0, o[nt][1] * f0);
                *reinterpret_cast<float2*>(ored + (warp * 16 + gr + 8) * DV + cc) =
                    make_float2(o[nt][2] * f1, o[nt][3] * f1);
            }
        }
        if (threadIdx.x < 16) {
            const int h = threadIdx.x;
            float M = -INFINITY;
            for (int w2 = 0; w2 < 4; ++w2) M = fmaxf(M, wm[w2][h]);
            float L = 0.f;
            for (int w2 = 0; w2 < 4; ++w2)
                if (wm[w2][h] != -INFINITY) L += wl[w2][h] * exp2f(wm[w2][h] - M);
            lse2s[br][h] = L > 0.f ? M + log2f(L) : -INFINITY;
            Lsum[h] = L;
        }
        __syncthreads();
        // dgate_h = <dO_h, o_c,h>, 8 threads per head; D_c = gate * dgate
        {
            const int h = threadIdx.x >> 3, part = threadIdx.x & 7;
            float acc = 0.f;
            const float L = Lsum[h];
            if (h < p.HG && L > 0.f) {
                const __nv_bfloat16* dor = reinterpret_cast<const __nv_bfloat16*>(dos + h * VP);
                for (int cc = part; cc < DV; cc += 8) {
                    const float oc = (ored[h * DV + cc] + ored[(16 + h) * DV + cc] + ored[(32 + h) * DV + cc] +
                                      ored[(48 + h) * DV + cc]) / L;
                    acc += oc * __bfloat162float(dor[cc]);
                }
            }
#pragma unroll
            for (int q2 = 1; q2 <= 4; q2 <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, q2);
            if (part == 0) {
                Ds[br][h] = gs[br][h] * acc;
                if (h < p.HG) {
                    p.dgates[(rowbase + h) * 3 + br] = acc;
                    p.lse2[(rowbase + h) * 3 + br] = lse2s[br][h];
                    p.dlt[(rowbase + h) * 3 + br] = gs[br][h] * acc;
                }
            }
        }
        __syncthreads();                                      // ored dead, staging free
    }

    // ---------------- pass 2, every branch: dS = P (g dP - D), dq += dS K
    float dq[DK / 8][4];
#pragma unroll
    for (int nt = 0; nt < DK / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) dq[nt][e] = 0.f;
    for (int br = 0; br < 3; ++br) {
        if (!((p.q_branches >> br) & 1)) continue;
        int lo;
        const int nk = branch_keys(br, lo);
        const int nch = (nk + 31) / 32;
        const float L0 = lse2s[br][gr], L1 = lse2s[br][gr + 8];
        const float D0 = Ds[br][gr], D1 = Ds[br][gr + 8];
        const float g0 = gs[br][gr], g1 = gs[br][gr + 8];
        for (int ch = warp; ch < nch; ch += 4) {
            const int k0 = ch * 32;
            const int nval = stage(br, lo, nk, k0);
            float sf[4][4], dp[4][4];
            warp_logits<DK>(qa, smem_u32(ks), sf);
            warp_logits_sa<DV>(smem_u32(dos), smem_u32(vs), dp);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const bool hi = e >= 2;
                    const float Lr = hi ? L1 : L0;
                    const bool ok = nt * 8 + tg * 2 + (e & 1) < nval && Lr != -INFINITY;
                    const float P = ok ? exp2f(sf[nt][e] * c - Lr) : 0.f;
                    sf[nt][e] = P * ((hi ? g1 : g0) * dp[nt][e] - (hi ? D1 : D0));
                }
            warp_pv<DK>(sf, smem_u32(ks), dq);
            __syncwarp();
        }
    }
    __syncthreads();
    // merge dq over the 4 warps, fixed order
    float* qred = reinterpret_cast<float*>(bsm);               // [4][16][DK]
#pragma unroll
    for (int nt = 0; nt < DK / 8; ++nt) {
        const int cc = nt * 8 + tg * 2;
        *reinterpret_cast<float2*>(qred + (warp * 16 + gr) * DK + cc) = make_float2(dq[nt][0], dq[nt][1]);
        *reinterpret_cast<float2*>(qred + (warp * 16 + gr + 8) * DK + cc) = make_float2(dq[nt][2], dq[nt][3]);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < p.HG * DK; e += 128) {
        const int h = e / DK, cc = e % DK;
        p.dq[(rowbase + h) * DK + cc] =
            p.scale * (qred[h * DK + cc] + qred[(16 + h) * DK + cc] + qred[(32 + h) * DK + cc] + qred[(48 + h) * DK + cc]);
    }
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
