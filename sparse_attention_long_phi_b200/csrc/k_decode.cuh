// k_decode.cuh -- batched decode step (page "硬件对齐+原生训练！DeepSeek NSA打造高效
// 稀疏Attention", 效率分析 解码速度: per step NSA reads the compressed tokens, the
// selected blocks and the window, not the whole cache).
//
// One query per sequence at t = L-1 over packed varlen caches.  The step is
// HBM-bound; the kernels stream each cache row once:
//   1. dec_cmp_partial  split-K over the compressed cache: logits for the HG
//                       heads of a group (kept for step 2), split max/sum and
//                       the split's P.V~.
//   2. dec_cmp_combine  merge the splits -> o_cmp and the row LSE; normalised
//                       compressed probabilities summed over heads, mapped to
//                       selection blocks; top-n by one warp -> sel_idx.
//   3. dec_slcwin_partial  one CTA per 64-token unit of (selected blocks U
//                       window blocks): logits once, partial softmax of the
//                       selected and window branches over the unit.
//   4. dec_final        merge units per branch; out = sum_c g_c o_c; lse.
#pragma once
#include "nsa_dev.cuh"
#include "k_topn.cuh"

namespace nsa {

constexpr int kDecCH = 128;    // compressed keys per split
constexpr int kDecUnit = 64;   // tokens per selected/window unit

struct DecParams {
    int S, H, G, HG, DK, DV;
    int l, d, lp, n, fi, fl, w;
    float scale_log2;
    const __nv_bfloat16 *q, *kcache, *vcache, *kccache, *vccache;
    const int64_t *kv_off, *cmp_off;
    const float* gates;
    float* out;
    int32_t* sel_idx;
    float* lse;
    float* logits;   // [S][G][16][Cmax]     log2-scaled logits
    float* part1;    // [S][G][NSPL][16][2+DV]
    float* ocmp;     // [S][G][16][DV]
    float* lsecmp;   // [S][G][16]            log2 units
    float* part2;    // [S][G][NU][2][16][2+DV]
    int Cmax, NSPL, NU, NSmax;
};

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&f)[8]) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = __bfloat162float(h[e]);
}

// q of the group's heads into shared memory as fp32 [16][DK] (rows >= HG zero)
__device__ __forceinline__ void dec_load_q(const DecParams& p, int s, int g, float* qs) {
    for (int e = threadIdx.x; e < 16 * p.DK; e += blockDim.x) {
        const int h = e / p.DK, c = e % p.DK;
        qs[e] = h < p.HG ? __bfloat162float(p.q[((size_t)s * p.H + g * p.HG + h) * p.DK + c]) : 0.f;
    }
}

// sorted union of the selected blocks and the blocks overlapping the window
__device__ __forceinline__ int dec_units(const DecParams& p, const int32_t* sel, int L, int* list) {
    const int wlo = max(0, L - p.w) / p.lp, whi = (L - 1) / p.lp;
    int i = 0, j = wlo, cnt = 0, last = -1;
    while (true) {
        const int a = (i < p.n && sel[i] >= 0) ? sel[i] : 0x7fffffff;
        const int b = j <= whi ? j : 0x7fffffff;
        const int m = min(a, b);
        if (m == 0x7fffffff) break;
        if (m == a) ++i;
        if (m == b) ++j;
        if (m != last) list[cnt++] = m;
        last = m;
    }
    return cnt;
}

// -------------------------------------------------------------- step 1
__global__ void __launch_bounds__(256) dec_cmp_partial(const DecParams p) {
    __shared__ float qs[16 * 192];
    __shared__ float Sm[16][kDecCH];
    const int sp = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
    const int64_t cbase = p.cmp_off[s];
    const int C = (int)(p.cmp_off[s + 1] - cbase);
    if (C > p.Cmax) {
        if (threadIdx.x == 0 && sp == 0) atomicOr(&g_nsa_error, 4u);
        return;
    }
    const int c0 = sp * kDecCH;
    if (c0 >= C) return;
    const int nk = min(kDecCH, C - c0);
    dec_load_q(p, s, g, qs);
    __syncthreads();
    {
        const int k = threadIdx.x & 127, hb = (threadIdx.x >> 7) * 8;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (k < nk) {
            const __nv_bfloat16* row = p.kccache + ((cbase + c0 + k) * p.G + g) * p.DK;
            for (int c = 0; c < p.DK; c += 8) {
                float kv[8];
                load8(row + c, kv);
#pragma unroll
                for (int h = 0; h < 8; ++h)
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[h] += qs[(hb + h) * p.DK + c + e] * kv[e];
            }
        }
        float* lg = p.logits + (((size_t)s * p.G + g) * 16) * p.Cmax;
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            const float v = k < nk ? acc[h] * p.scale_log2 : -INFINITY;
            Sm[hb + h][k] = v;
            if (k < nk) lg[(size_t)(hb + h) * p.Cmax + c0 + k] = v;
        }
    }
    __syncthreads();
    const int h = threadIdx.x >> 4, sub = threadIdx.x & 15;
    float m = -INFINITY;
    for (int k = sub; k < kDecCH; k += 16) m = fmaxf(m, Sm[h][k]);
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    for (int k = sub; k < kDecCH; k += 16) {
        const float e = Sm[h][k] == -INFINITY ? 0.f : exp2f(Sm[h][k] - m);
        Sm[h][k] = e;
        l += e;
    }
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    __syncthreads();
    // P.V~: thread (h, channel group)
    const int cw = p.DV / 16, cg = sub;
    float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < nk; ++k) {
        const float pk = Sm[h][k];
        const __nv_bfloat16* vr = p.vccache + ((cbase + c0 + k) * p.G + g) * p.DV + cg * cw;
        if (cw == 8) {
            float vv[8];
            load8(vr, vv);
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] += pk * vv[e];
        } else {
            for (int e = 0; e < cw; ++e) o[e] += pk * __bfloat162float(vr[e]);
        }
    }
    float* dst = p.part1 + ((((size_t)s * p.G + g) * p.NSPL + sp) * 16 + h) * (2 + p.DV);
    if (sub == 0) {
        dst[0] = m;
        dst[1] = l;
    }
    for (int e = 0; e < cw; ++e) dst[2 + cg * cw + e] = o[e];
}

// -------------------------------------------------------------- step 2
__global__ void __launch_bounds__(256) dec_cmp_combine(const DecParams p) {
    extern __shared__ float dsm[];
    float* psum = dsm;                    // [Cmax]
    float* pg = dsm + p.Cmax;             // [NSmax]
    __shared__ float lse2[16];
    const int g = blockIdx.x, s = blockIdx.y;
    const int64_t cbase = p.cmp_off[s];
    const int C = (int)(p.cmp_off[s + 1] - cbase);
    const int L = (int)(p.kv_off[s + 1] - p.kv_off[s]);
    const int t = L - 1;
    if (C > p.Cmax || L <= 0) return;
    const int nspl = (C + kDecCH - 1) / kDecCH;
    const int h = threadIdx.x >> 4, sub = threadIdx.x & 15;
    const float* part = p.part1 + (((size_t)s * p.G + g) * p.NSPL) * 16 * (2 + p.DV);
    float M = -INFINITY;
    for (int i = 0; i < nspl; ++i) M = fmaxf(M, part[((size_t)i * 16 + h) * (2 + p.DV)]);
    float Lsum = 0.f;
    for (int i = 0; i < nspl; ++i) {
        const float* pr = part + ((size_t)i * 16 + h) * (2 + p.DV);
        if (pr[0] != -INFINITY) Lsum += pr[1] * exp2f(pr[0] - M);
    }
    const int cw = p.DV / 16;
    for (int e = 0; e < cw; ++e) {
        const int c = sub * cw + e;
        float acc = 0.f;
        for (int i = 0; i < nspl; ++i) {
            const float* pr = part + ((size_t)i * 16 + h) * (2 + p.DV);
            if (pr[0] != -INFINITY) acc += pr[2 + c] * exp2f(pr[0] - M);
        }
        p.ocmp[(((size_t)s * p.G + g) * 16 + h) * p.DV + c] = Lsum > 0.f ? acc / Lsum : 0.f;
    }
    const float l2 = Lsum > 0.f ? M + log2f(Lsum) : -INFINITY;
    if (sub == 0) {
        lse2[h] = l2;
        p.lsecmp[((size_t)s * p.G + g) * 16 + h] = l2;
    }
    __syncthreads();
    // compressed probabilities summed over the group's heads
    const float* lg = p.logits + (((size_t)s * p.G + g) * 16) * p.Cmax;
    for (int i = threadIdx.x; i < C; i += blockDim.x) {
        float acc = 0.f;
        for (int hh = 0; hh < p.HG; ++hh)
            if (lse2[hh] != -INFINITY) acc += exp2f(lg[(size_t)hh * p.Cmax + i] - lse2[hh]);
        psum[i] = acc;
    }
    __syncthreads();
    // mapped to selection blocks with the overlap weights
    const int cps = p.l / p.d, spb = p.lp / p.d;
    const int NSs = (L + p.lp - 1) / p.lp;
    for (int j = threadIdx.x; j < NSs; j += blockDim.x) {
        float acc = 0.f;
        for (int i = j * spb - cps + 1; i <= j * spb + spb - 1; ++i) {
            if (i < 0 || i >= C) continue;
            int wgt = 0;
            for (int u = 0; u < cps; ++u) wgt += ((i + u) / spb == j);
            acc += (float)wgt * psum[i];
        }
        pg[j] = acc;
    }
    __syncthreads();
    if (threadIdx.x < 32)
        topn_row_warp(pg, t, p.n, p.lp, p.fi, p.fl, p.sel_idx + ((size_t)s * p.G + g) * p.n,
                      threadIdx.x);
}

// -------------------------------------------------------------- step 3
__global__ void __launch_bounds__(256) dec_slcwin_partial(const DecParams p) {
    __shared__ float qs[16 * 192];
    __shared__ float Sm[16][kDecUnit];
    __shared__ float P0[16][kDecUnit], P1[16][kDecUnit];
    __shared__ int list[48];
    __shared__ int nlist;
    const int ui = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
    const int64_t kb = p.kv_off[s];
    const int L = (int)(p.kv_off[s + 1] - kb);
    if (L <= 0) return;
    const int32_t* sel = p.sel_idx + ((size_t)s * p.G + g) * p.n;
    if (threadIdx.x == 0) nlist = dec_units(p, sel, L, list);
    __syncthreads();
    if (ui >= nlist) return;
    const int blk = list[ui];
    bool in_sel = false;
    for (int a = 0; a < p.n; ++a) in_sel |= (sel[a] == blk);
    dec_load_q(p, s, g, qs);
    __syncthreads();
    {
        const int k = threadIdx.x & 63, hb = (threadIdx.x >> 6) * 4;
        const int u = blk * p.lp + k;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (u < L) {
            const __nv_bfloat16* row = p.kcache + ((kb + u) * p.G + g) * p.DK;
            for (int c = 0; c < p.DK; c += 8) {
                float kv[8];
                load8(row + c, kv);
#pragma unroll
                for (int h = 0; h < 4; ++h)
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[h] += qs[(hb + h) * p.DK + c + e] * kv[e];
            }
        }
#pragma unroll
        for (int h = 0; h < 4; ++h) Sm[hb + h][k] = u < L ? acc[h] * p.scale_log2 : -INFINITY;
    }
    __syncthreads();
    const int h = threadIdx.x >> 4, sub = threadIdx.x & 15;
    float mb[2], lb[2];
#pragma unroll
    for (int br = 0; br < 2; ++br) {
        float m = -INFINITY;
        for (int k = sub; k < kDecUnit; k += 16) {
            const int u = blk * p.lp + k;
            const bool f = br == 0 ? (in_sel && u < L) : (u < L && u >= L - p.w);
            if (f) m = fmaxf(m, Sm[h][k]);
        }
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        for (int k = sub; k < kDecUnit; k += 16) {
            const int u = blk * p.lp + k;
            const bool f = br == 0 ? (in_sel && u < L) : (u < L && u >= L - p.w);
            const float e = (f && m != -INFINITY) ? exp2f(Sm[h][k] - m) : 0.f;
            (br == 0 ? P0 : P1)[h][k] = e;
            l += e;
        }
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        mb[br] = m;
        lb[br] = l;
    }
    __syncthreads();
    const int cw = p.DV / 16, cg = sub;
    float o0[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, o1[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const int nk = min(kDecUnit, L - blk * p.lp);
    for (int k = 0; k < nk; ++k) {
        const float a0 = P0[h][k], a1 = P1[h][k];
        const __nv_bfloat16* vr = p.vcache + ((kb + blk * p.lp + k) * p.G + g) * p.DV + cg * cw;
        if (cw == 8) {
            float vv[8];
            load8(vr, vv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                o0[e] += a0 * vv[e];
                o1[e] += a1 * vv[e];
            }
        } else {
            for (int e = 0; e < cw; ++e) {
                const float vv = __bfloat162float(vr[e]);
                o0[e] += a0 * vv;
                o1[e] += a1 * vv;
            }
        }
    }
#pragma unroll
    for (int br = 0; br < 2; ++br) {
        float* dst = p.part2 + (((((size_t)s * p.G + g) * p.NU + ui) * 2 + br) * 16 + h) * (2 + p.DV);
        if (sub == 0) {
            dst[0] = mb[br];
            dst[1] = lb[br];
        }
        for (int e = 0; e < cw; ++e) dst[2 + cg * cw + e] = br == 0 ? o0[e] : o1[e];
    }
}

// -------------------------------------------------------------- step 4
__global__ void __launch_bounds__(256) dec_final(const DecParams p) {
    __shared__ int list[48];
    __shared__ int nlist;
    const int g = blockIdx.x, s = blockIdx.y;
    const int L = (int)(p.kv_off[s + 1] - p.kv_off[s]);
    if (L <= 0) return;
    const int32_t* sel = p.sel_idx + ((size_t)s * p.G + g) * p.n;
    if (threadIdx.x == 0) nlist = dec_units(p, sel, L, list);
    __syncthreads();
    const int h = threadIdx.x >> 4, sub = threadIdx.x & 15;
    const int cw = p.DV / 16;
    float Mb[2], Lb[2];
#pragma unroll
    for (int br = 0; br < 2; ++br) {
        float M = -INFINITY;
        for (int u = 0; u < nlist; ++u)
            M = fmaxf(M, p.part2[(((((size_t)s * p.G + g) * p.NU + u) * 2 + br) * 16 + h) * (2 + p.DV)]);
        float Ls = 0.f;
        for (int u = 0; u < nlist; ++u) {
            const float* pr = p.part2 + (((((size_t)s * p.G + g) * p.NU + u) * 2 + br) * 16 + h) * (2 + p.DV);
            if (pr[0] != -INFINITY) Ls += pr[1] * exp2f(pr[0] - M);
        }
        Mb[br] = M;
        Lb[br] = Ls;
    }
    if (h < p.HG) {
        const size_t row = (size_t)s * p.H + g * p.HG + h;
        const float g0 = p.gates[row * 3 + 0], g1 = p.gates[row * 3 + 1], g2 = p.gates[row * 3 + 2];
        for (int e = 0; e < cw; ++e) {
            const int c = sub * cw + e;
            float ob[2];
#pragma unroll
            for (int br = 0; br < 2; ++br) {
                float acc = 0.f;
                for (int u = 0; u < nlist; ++u) {
                    const float* pr = p.part2 + (((((size_t)s * p.G + g) * p.NU + u) * 2 + br) * 16 + h) * (2 + p.DV);
                    if (pr[0] != -INFINITY) acc += pr[2 + c] * exp2f(pr[0] - Mb[br]);
                }
                ob[br] = Lb[br] > 0.f ? acc / Lb[br] : 0.f;
            }
            const float oc = p.ocmp[(((size_t)s * p.G + g) * 16 + h) * p.DV + c];
            p.out[row * p.DV + c] = g0 * oc + g1 * ob[0] + g2 * ob[1];
        }
        if (sub == 0 && p.lse) {
            const float lc = p.lsecmp[((size_t)s * p.G + g) * 16 + h];
            p.lse[row * 3 + 0] = lc == -INFINITY ? -INFINITY : lc * kLn2;
            p.lse[row * 3 + 1] = Lb[0] > 0.f ? (Mb[0] + log2f(Lb[0])) * kLn2 : -INFINITY;
            p.lse[row * 3 + 2] = Lb[1] > 0.f ? (Mb[1] + log2f(Lb[1])) * kLn2 : -INFINITY;
        }
    }
}

// workspace bytes for S sequences of at most Lmax tokens
inline size_t decode_ws_bytes(int64_t S, int64_t Lmax, int64_t G, int64_t l, int64_t d, int64_t lp,
                              int64_t w, int64_t n, int64_t DV) {
    const int64_t Cmax = Lmax >= l ? (Lmax - l) / d + 1 : 1;
    const int64_t NSPL = (Cmax + kDecCH - 1) / kDecCH;
    const int64_t NU = n + (w + lp - 1) / lp + 1;
    auto a = [](size_t x) { return (x + 255) & ~size_t(255); };
    size_t o = 0;
    o += a((size_t)S * G * 16 * Cmax * 4);
    o += a((size_t)S * G * NSPL * 16 * (2 + DV) * 4);
    o += a((size_t)S * G * 16 * DV * 4);
    o += a((size_t)S * G * 16 * 4);
    o += a((size_t)S * G * NU * 2 * 16 * (2 + DV) * 4);
    return o;
}

}  // namespace nsa
