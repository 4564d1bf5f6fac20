// k_decode.cuh -- batched decode step (page "硬件对齐+原生训练！DeepSeek NSA打造高效
// 稀疏Attention", 效率分析 解码速度: per step NSA reads the compressed tokens, the
// selected blocks and the window, not the whole cache).
//
// One query per sequence at t = L-1 over packed varlen caches.  The step is
// HBM-bound; every cache row is read once, with 16-byte coalesced loads into
// shared memory, and the 16 heads of a GQA group are the M = 16 side of
// warp-level bf16 tensor-core products (mma.sync m16n8k16, fp32 accumulate):
//   1. dec_cmp_partial  split-K over the compressed cache (128 keys per CTA,
//                       32 per warp): logits, split max / sum, P.V~, and the
//                       per-head selection-block sums of exp(logit - split max)
//                       (mapped with the overlap weights), so the scores can be
//                       normalised exactly once the row LSE is known.
//   2. dec_cmp_combine  merge the splits -> o_cmp and the row LSE; group
//                       importance scores = sum over heads and splits of the
//                       block sums rescaled by exp(split max - LSE); top-n by
//                       one warp -> sel_idx.
//   3. dec_slcwin_partial  one CTA per 64-token unit of (selected blocks U
//                       window blocks): logits once, partial softmax of the
//                       selected and window branches over the unit.
//   4. dec_final        merge units per branch; out = sum_c g_c o_c; lse.
#pragma once
#include "nsa_dev.cuh"
#include "k_topn.cuh"
#include "k_mma.cuh"

namespace nsa {

constexpr int kDecCH = 128;     // compressed keys per split (4 warps x 32)
constexpr int kDecUnit = 64;    // tokens per selected/window unit (2 warps x 32)
constexpr int kDecNJB = 132;    // block-score slots per split (>= 128/SPB + 1)
constexpr int kDecWJB = 34;     // block-score slots per warp of 32 keys (>= 32/SPB + 2)
constexpr int kDecMaxSplits = 64;  // compressed-cache splits per sequence (Lmax <= 8192 * 16 + l)

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
    float* part1;    // [S][G][NSPL][16][2+DV]   split max (log2 units), sum, unnormalised O
    float* bsc;      // [S][G][NSPL][16][kDecNJB] block sums of exp2(s - split max)
    float* ocmp;     // [S][G][16][DV]
    float* lsecmp;   // [S][G][16]               log2 units
    float* part2;    // [S][G][NU][2][16][2+DV]
    int Cmax, NSPL, NU, NSmax;
};

// Q of the group's 16 heads (rows >= HG zero) as A fragments for DK/16 k-steps
template <int DK>
__device__ __forceinline__ void load_q_frags(const DecParams& p, int s, int g, uint32_t (&qa)[DK / 16][4]) {
    const int lane = threadIdx.x & 31, gr = lane >> 2, tg = lane & 3;
    const __nv_bfloat16* q = p.q + ((size_t)s * p.H + (size_t)g * p.HG) * DK;
#pragma unroll
    for (int kk = 0; kk < DK / 16; ++kk) {
        const int c = kk * 16 + tg * 2;
        auto ld = [&](int row, int col) -> uint32_t {
            return row < p.HG ? *reinterpret_cast<const uint32_t*>(q + (size_t)row * DK + col) : 0u;
        };
        qa[kk][0] = ld(gr, c);
        qa[kk][1] = ld(gr + 8, c);
        qa[kk][2] = ld(gr, c + 8);
        qa[kk][3] = ld(gr + 8, c + 8);
    }
}

// -------------------------------------------------------------- step 1
template <int DK, int DV>
__global__ void __launch_bounds__(128) dec_cmp_partial(const DecParams p) {
    constexpr int KP = DK * 2 + 16, VP = DV * 2 + 16;
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ float redm[4][16], redl[4][16];
    __shared__ float bsw[4][16][kDecWJB];
    const int sp = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gr = lane >> 2, tg = lane & 3;
    const int64_t cbase = p.cmp_off[s];
    const int C = (int)(p.cmp_off[s + 1] - cbase);
    if (C > p.Cmax) {
        if (threadIdx.x == 0 && sp == 0) atomicOr(&g_nsa_error, 4u);
        return;
    }
    const int c0 = sp * kDecCH;
    if (c0 >= C) return;
    uint8_t* ks = dsm + warp * 32 * (KP + VP);
    uint8_t* vs = ks + 32 * KP;
    const int k0 = c0 + warp * 32;                       // first key of this warp
    const int nval = max(0, min(32, C - k0));
    warp_copy_rows(ks, KP, p.kccache + ((cbase + k0) * p.G + g) * DK, (size_t)p.G * DK, 32, nval, DK);
    warp_copy_rows(vs, VP, p.vccache + ((cbase + k0) * p.G + g) * DV, (size_t)p.G * DV, 32, nval, DV);
    uint32_t qa[DK / 16][4];
    load_q_frags<DK>(p, s, g, qa);
    cp_async_wait();
    __syncwarp();
    float sf[4][4];
    warp_logits<DK>(qa, smem_u32(ks), sf);
    // scale, mask keys past the cache, warp max per head row (rows gr, gr+8)
    float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int key = nt * 8 + tg * 2 + (e & 1);
            float v = key < nval ? sf[nt][e] * p.scale_log2 : -INFINITY;
            sf[nt][e] = v;
            if (e < 2) m0 = fmaxf(m0, v);
            else m1 = fmaxf(m1, v);
        }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
    }
    if (tg == 0) {
        redm[warp][gr] = m0;
        redm[warp][gr + 8] = m1;
    }
    __syncthreads();
    m0 = fmaxf(fmaxf(redm[0][gr], redm[1][gr]), fmaxf(redm[2][gr], redm[3][gr]));
    m1 = fmaxf(fmaxf(redm[0][gr + 8], redm[1][gr + 8]), fmaxf(redm[2][gr + 8], redm[3][gr + 8]));
    // P = exp2(s - split max); row sums; per-head block sums (overlap weights)
    const int cps = p.l / p.d, spb = p.lp / p.d;
    const int nj = kDecCH / spb + (cps + spb - 2) / spb + 1;   // blocks this split touches
    for (int e = lane; e < 16 * kDecWJB; e += 32) bsw[warp][e / kDecWJB][e % kDecWJB] = 0.f;
    const int wj0 = (warp * 32) / spb;                        // first block this warp touches
    __syncwarp();
    float l0 = 0.f, l1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float mm = e < 2 ? m0 : m1;
            const float pv = sf[nt][e] == -INFINITY ? 0.f : exp2f(sf[nt][e] - mm);
            sf[nt][e] = pv;
            if (e < 2) l0 += pv;
            else l1 += pv;
        }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    // block sums: lanes of a quad own disjoint keys of the same two heads;
    // accumulate per key in a fixed order (deterministic)
    for (int q = 0; q < 4; ++q) {
        if (tg == q) {
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int kl = nt * 8 + tg * 2 + (e & 1);
                    const int row = e < 2 ? gr : gr + 8;
                    const int ig = warp * 32 + kl;            // key index within the split
                    for (int u = 0; u < cps; ++u) {
                        const int jl = (ig + u) / spb - wj0;
                        bsw[warp][row][jl] += sf[nt][e];
                    }
                }
        }
        __syncwarp();
    }
    if (tg == 0) {
        redl[warp][gr] = l0;
        redl[warp][gr + 8] = l1;
    }
    // P.V~ of this warp's keys
    float o[DV / 8][4];
#pragma unroll
    for (int nt = 0; nt < DV / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
    warp_pv<DV>(sf, smem_u32(vs), o);
    __syncthreads();
    // sum the 4 warps' O in shared memory (reusing the staging area), fixed order
    float* ored = reinterpret_cast<float*>(dsm);          // [4][16][DV]
#pragma unroll
    for (int nt = 0; nt < DV / 8; ++nt) {
        const int ch = nt * 8 + tg * 2;
        ored[(warp * 16 + gr) * DV + ch] = o[nt][0];
        ored[(warp * 16 + gr) * DV + ch + 1] = o[nt][1];
        ored[(warp * 16 + gr + 8) * DV + ch] = o[nt][2];
        ored[(warp * 16 + gr + 8) * DV + ch + 1] = o[nt][3];
    }
    __syncthreads();
    float* dst = p.part1 + (((size_t)s * p.G + g) * p.NSPL + sp) * 16 * (2 + DV);
    for (int e = threadIdx.x; e < 16 * DV; e += 128) {
        const int h = e / DV, c = e % DV;
        dst[h * (2 + DV) + 2 + c] = ored[h * DV + c] + ored[(16 + h) * DV + c] + ored[(32 + h) * DV + c] +
                                    ored[(48 + h) * DV + c];
    }
    if (threadIdx.x < 16) {
        const int h = threadIdx.x;
        dst[h * (2 + DV)] = fmaxf(fmaxf(redm[0][h], redm[1][h]), fmaxf(redm[2][h], redm[3][h]));
        dst[h * (2 + DV) + 1] = redl[0][h] + redl[1][h] + redl[2][h] + redl[3][h];
    }
    float* bdst = p.bsc + (((size_t)s * p.G + g) * p.NSPL + sp) * 16 * kDecNJB;
    for (int e = threadIdx.x; e < 16 * kDecNJB; e += 128) {
        const int h = e / kDecNJB, j = e % kDecNJB;
        float acc = 0.f;
        if (j < nj) {
#pragma unroll
            for (int w2 = 0; w2 < 4; ++w2) {      // fixed order: deterministic
                const int jl = j - (w2 * 32) / spb;
                if (jl >= 0 && jl < kDecWJB) acc += bsw[w2][h][jl];
            }
        }
        bdst[e] = acc;
    }
}

// -------------------------------------------------------------- step 2
template <int DV>
__global__ void __launch_bounds__(256) dec_cmp_combine(const DecParams p) {
    extern __shared__ float pg[];                      // [NSmax]
    __shared__ float lse2[16];
    __shared__ float fac[kDecMaxSplits][16];           // per split scale exp2(m_split - LSE)
    const int g = blockIdx.x, s = blockIdx.y;
    const int64_t cbase = p.cmp_off[s];
    const int C = (int)(p.cmp_off[s + 1] - cbase);
    const int L = (int)(p.kv_off[s + 1] - p.kv_off[s]);
    const int t = L - 1;
    if (C > p.Cmax || L <= 0) return;
    const int nspl = (C + kDecCH - 1) / kDecCH;
    const float* part = p.part1 + (((size_t)s * p.G + g) * p.NSPL) * 16 * (2 + DV);
    if (threadIdx.x < 16) {
        const int h = threadIdx.x;
        float M = -INFINITY;
        for (int i = 0; i < nspl; ++i) M = fmaxf(M, part[((size_t)i * 16 + h) * (2 + DV)]);
        float Ls = 0.f;
        for (int i = 0; i < nspl; ++i) {
            const float* pr = part + ((size_t)i * 16 + h) * (2 + DV);
            if (pr[0] != -INFINITY) Ls += pr[1] * exp2f(pr[0] - M);
        }
        const float l2 = Ls > 0.f ? M + log2f(Ls) : -INFINITY;
        lse2[h] = l2;
        p.lsecmp[((size_t)s * p.G + g) * 16 + h] = l2;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < nspl * 16; e += blockDim.x) {
        const int i = e / 16, h = e % 16;
        const float m = part[((size_t)i * 16 + h) * (2 + DV)];
        fac[i][h] = (h < p.HG && m != -INFINITY && lse2[h] != -INFINITY) ? exp2f(m - lse2[h]) : 0.f;
    }
    __syncthreads();
    // o_cmp = sum_i O_i * exp2(m_i - LSE)
    for (int e = threadIdx.x; e < 16 * DV; e += blockDim.x) {
        const int h = e / DV, c = e % DV;
        float acc = 0.f;
        for (int i = 0; i < nspl; ++i) acc += part[((size_t)i * 16 + h) * (2 + DV) + 2 + c] * fac[i][h];
        p.ocmp[(((size_t)s * p.G + g) * 16 + h) * DV + c] = acc;
    }
    // group scores: block j lies in split j / (128/spb) and, through the
    // overlap of its last compressed block, in the split before it
    const int spb = p.lp / p.d;
    const int per = kDecCH / spb;
    const int NSs = (L + p.lp - 1) / p.lp;
    const float* bs = p.bsc + (((size_t)s * p.G + g) * p.NSPL) * 16 * kDecNJB;
    for (int j = threadIdx.x; j < NSs; j += blockDim.x) {
        float acc = 0.f;
        for (int i = max(0, j / per - 1); i <= min(nspl - 1, j / per); ++i) {
            const int jl = j - i * per;
            if (jl < 0 || jl >= kDecNJB) continue;
            for (int h = 0; h < p.HG; ++h) acc += bs[((size_t)i * 16 + h) * kDecNJB + jl] * fac[i][h];
        }
        pg[j] = acc;
    }
    __syncthreads();
    if (threadIdx.x < 32)
        topn_row_warp(pg, t, p.n, p.lp, p.fi, p.fl, p.sel_idx + ((size_t)s * p.G + g) * p.n, threadIdx.x);
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

// -------------------------------------------------------------- step 3
template <int DK, int DV>
__global__ void __launch_bounds__(64) dec_slcwin_partial(const DecParams p) {
    constexpr int KP = DK * 2 + 16, VP = DV * 2 + 16;
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ float red[2][2][2][16];     // [branch][max|sum][warp][head]
    __shared__ int list[48];
    __shared__ int nlist;
    const int ui = blockIdx.x, g = blockIdx.y, s = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gr = lane >> 2, tg = lane & 3;
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
    uint8_t* ks = dsm + warp * 32 * (KP + VP);
    uint8_t* vs = ks + 32 * KP;
    const int u0 = blk * p.lp + warp * 32;                    // first token of this warp
    const int nval = max(0, min(32, L - u0));
    warp_copy_rows(ks, KP, p.kcache + ((kb + u0) * p.G + g) * DK, (size_t)p.G * DK, 32, nval, DK);
    warp_copy_rows(vs, VP, p.vcache + ((kb + u0) * p.G + g) * DV, (size_t)p.G * DV, 32, nval, DV);
    uint32_t qa[DK / 16][4];
    load_q_frags<DK>(p, s, g, qa);
    cp_async_wait();
    __syncwarp();
    float sf[4][4];
    warp_logits<DK>(qa, smem_u32(ks), sf);
    float mx[2][2];
#pragma unroll
    for (int br = 0; br < 2; ++br) mx[br][0] = mx[br][1] = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int u = u0 + nt * 8 + tg * 2 + (e & 1);
            const float v = u < L ? sf[nt][e] * p.scale_log2 : -INFINITY;
            sf[nt][e] = v;
            if (in_sel) mx[0][e >> 1] = fmaxf(mx[0][e >> 1], v);
            if (u >= L - p.w) mx[1][e >> 1] = fmaxf(mx[1][e >> 1], v);
        }
#pragma unroll
    for (int br = 0; br < 2; ++br)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int o = 1; o <= 2; o <<= 1) mx[br][hf] = fmaxf(mx[br][hf], __shfl_xor_sync(0xffffffffu, mx[br][hf], o));
    if (tg == 0) {
#pragma unroll
        for (int br = 0; br < 2; ++br) {
            red[br][0][warp][gr] = mx[br][0];
            red[br][0][warp][gr + 8] = mx[br][1];
        }
    }
    __syncthreads();
#pragma unroll
    for (int br = 0; br < 2; ++br) {
        mx[br][0] = fmaxf(red[br][0][0][gr], red[br][0][1][gr]);
        mx[br][1] = fmaxf(red[br][0][0][gr + 8], red[br][0][1][gr + 8]);
    }
    float ls[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    float o[2][DV / 8][4];
#pragma unroll
    for (int br = 0; br < 2; ++br) {
        float pf[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int u = u0 + nt * 8 + tg * 2 + (e & 1);
                const bool f = br == 0 ? (in_sel && u < L) : (u < L && u >= L - p.w);
                const float m = mx[br][e >> 1];
                const float pv = (f && m != -INFINITY) ? exp2f(sf[nt][e] - m) : 0.f;
                pf[nt][e] = pv;
                ls[br][e >> 1] += pv;
            }
#pragma unroll
        for (int nt = 0; nt < DV / 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[br][nt][e] = 0.f;
        warp_pv<DV>(pf, smem_u32(vs), o[br]);
    }
#pragma unroll
    for (int br = 0; br < 2; ++br)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
            for (int q2 = 1; q2 <= 2; q2 <<= 1) ls[br][hf] += __shfl_xor_sync(0xffffffffu, ls[br][hf], q2);
    if (tg == 0) {
#pragma unroll
        for (int br = 0; br < 2; ++br) {
            red[br][1][warp][gr] = ls[br][0];
            red[br][1][warp][gr + 8] = ls[br][1];
        }
    }
    __syncthreads();
    float* ored = reinterpret_cast<float*>(dsm);            // [2 br][2 warps][16][DV]
#pragma unroll
    for (int br = 0; br < 2; ++br)
#pragma unroll
        for (int nt = 0; nt < DV / 8; ++nt) {
            const int ch = nt * 8 + tg * 2;
            float* base = ored + ((br * 2 + warp) * 16) * DV;
            base[gr * DV + ch] = o[br][nt][0];
            base[gr * DV + ch + 1] = o[br][nt][1];
            base[(gr + 8) * DV + ch] = o[br][nt][2];
            base[(gr + 8) * DV + ch + 1] = o[br][nt][3];
        }
    __syncthreads();
#pragma unroll
    for (int br = 0; br < 2; ++br) {
        float* dst = p.part2 + (((((size_t)s * p.G + g) * p.NU + ui) * 2 + br) * 16) * (2 + DV);
        for (int e = threadIdx.x; e < 16 * DV; e += 64) {
            const int h = e / DV, c = e % DV;
            dst[h * (2 + DV) + 2 + c] = ored[((br * 2 + 0) * 16 + h) * DV + c] + ored[((br * 2 + 1) * 16 + h) * DV + c];
        }
        if (threadIdx.x < 16) {
            const int h = threadIdx.x;
            dst[h * (2 + DV)] = fmaxf(red[br][0][0][h], red[br][0][1][h]);
            dst[h * (2 + DV) + 1] = red[br][1][0][h] + red[br][1][1][h];
        }
    }
}

// -------------------------------------------------------------- step 4
template <int DV>
__global__ void __launch_bounds__(256) dec_final(const DecParams p) {
    __shared__ int list[48];
    __shared__ int nlist;
    __shared__ float fac[2][48][16];
    __shared__ float Lb[2][16];
    const int g = blockIdx.x, s = blockIdx.y;
    const int L = (int)(p.kv_off[s + 1] - p.kv_off[s]);
    if (L <= 0) return;
    const int32_t* sel = p.sel_idx + ((size_t)s * p.G + g) * p.n;
    if (threadIdx.x == 0) nlist = dec_units(p, sel, L, list);
    __syncthreads();
    const float* part = p.part2 + ((((size_t)s * p.G + g) * p.NU) * 2) * 16 * (2 + DV);
    if (threadIdx.x < 32) {
        const int br = threadIdx.x / 16, h = threadIdx.x % 16;
        float M = -INFINITY;
        for (int u = 0; u < nlist; ++u) M = fmaxf(M, part[(((size_t)u * 2 + br) * 16 + h) * (2 + DV)]);
        float Ls = 0.f;
        for (int u = 0; u < nlist; ++u) {
            const float* pr = part + (((size_t)u * 2 + br) * 16 + h) * (2 + DV);
            const float f = pr[0] != -INFINITY ? exp2f(pr[0] - M) : 0.f;
            fac[br][u][h] = f;
            Ls += pr[1] * f;
        }
        Lb[br][h] = Ls;
        if (h < p.HG && p.lse) {
            const size_t row = (size_t)s * p.H + g * p.HG + h;
            p.lse[row * 3 + 1 + br] = Ls > 0.f ? (M + log2f(Ls)) * kLn2 : -INFINITY;
            if (br == 0) {
                const float lc = p.lsecmp[((size_t)s * p.G + g) * 16 + h];
                p.lse[row * 3] = lc == -INFINITY ? -INFINITY : lc * kLn2;
            }
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < p.HG * DV; e += blockDim.x) {
        const int h = e / DV, c = e % DV;
        float ob[2];
#pragma unroll
        for (int br = 0; br < 2; ++br) {
            float acc = 0.f;
            for (int u = 0; u < nlist; ++u) acc += part[(((size_t)u * 2 + br) * 16 + h) * (2 + DV) + 2 + c] * fac[br][u][h];
            ob[br] = Lb[br][h] > 0.f ? acc / Lb[br][h] : 0.f;
        }
        const size_t row = (size_t)s * p.H + g * p.HG + h;
        const float oc = p.ocmp[(((size_t)s * p.G + g) * 16 + h) * DV + c];   // normalised
        p.out[row * DV + c] = p.gates[row * 3] * oc + p.gates[row * 3 + 1] * ob[0] + p.gates[row * 3 + 2] * ob[1];
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
    o += a((size_t)S * G * NSPL * 16 * (2 + DV) * 4);
    o += a((size_t)S * G * NSPL * 16 * kDecNJB * 4);
    o += a((size_t)S * G * 16 * DV * 4);
    o += a((size_t)S * G * 16 * 4);
    o += a((size_t)S * G * NU * 2 * 16 * (2 + DV) * 4);
    return o;
}

}  // namespace nsa
