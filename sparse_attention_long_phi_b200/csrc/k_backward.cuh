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
// Kernels (SIMT, fp32 accumulation):
//   bwd_query_mma        one CTA per (b, t, g) on warp-level bf16 tensor cores
//                        (the 16 heads of the group are the M side): pass 1
//                        recomputes every branch's LSE and o_c (online softmax
//                        per warp, merged across warps) and writes dgates and
//                        D_c; pass 2 recomputes S and dP = dO_c V^T, forms dS
//                        and accumulates dq = scale dS K.
//   bwd_kv_mma<BR>       key-centric: a tile of 64 keys (raw tokens for the
//                        window and selected branches, compressed blocks for
//                        the compressed one) accumulates over the queries that
//                        read it, then adds into dk/dv (dK~/dV~) atomically.
//                        Selected keys find their queries through an inverse
//                        index (block -> tokens) built by count / scan / fill.
//   bwd_phiT_kernel      dk/dv += phi^T(dK~/dV~).
#pragma once
#include "nsa_dev.cuh"
#include "k_mma.cuh"

namespace nsa {

enum { kBrCmp = 0, kBrSlc = 1, kBrWin = 2 };
constexpr int kBwdChunk = 128;     // tokens per key-centric work item

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
    for (int br = 0; br < 3; ++br) {
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

// --------------------------------------------------------- per key tile
// One CTA of 4 warps = 64 keys (warp w: keys 16w..16w+15 of the tile) and a
// run of up to kBwdChunk tokens that attend them; per token, on warp-level
// bf16 tensor cores (mma.sync m16n8k16) with the 16 heads as the N side:
//   S^T = K_w Q_t^T,  dP^T = V_w dO_t^T                 (16 keys x 16 heads)
//   P = exp(S - LSE_h), dS = P (g_h dP - D_h)
//   dK_w += scale dS^T Q_t,  dV_w += (g P)^T dO_t       (in registers)
// The tile's K/V rows and the tokens' Q/dO rows (double-buffered) sit in
// shared memory; dK/dV are added to the fp32 outputs once at the end.
// grid.z = b*G + g.  WIN: grid (key tiles of 64 tokens, token chunks).
// CMP: grid (key tiles of 64 compressed blocks, token chunks).
// SLC: grid.x = chunk id over the inverse index (binary search), b and g
// from the entry found.
template <int DK, int DV>
__host__ __device__ constexpr int bwd_kv_mma_smem() {
    return 64 * ((DK * 2 + 16) + (DV * 2 + 16)) + 2 * 16 * ((DK * 2 + 16) + (DV * 2 + 16));
}

template <int DK, int DV, int BR>
__global__ void __launch_bounds__(128) bwd_kv_mma(const BwdParams p) {
    constexpr int KP = DK * 2 + 16, VP = DV * 2 + 16;
    extern __shared__ __align__(16) uint8_t bsm[];
    uint8_t* kt = bsm;                          // [64][KP]
    uint8_t* vt = kt + 64 * KP;                 // [64][VP]
    uint8_t* tokb = vt + 64 * VP;               // 2 x ([16][KP] Q rows, [16][VP] dO rows)
    __shared__ float sl[2][16], sD[2][16], sg[2][16];
    __shared__ int stok[2];
    int b = blockIdx.z / p.G, g = blockIdx.z % p.G;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gr = lane >> 2, tg = lane & 3;

    int key0, tok_lo, tok_hi;           // keys key0..key0+63; tokens (or list entries) [tok_lo, tok_hi)
    const int* toklist = nullptr;
    if (BR == kBrSlc) {
        const int cid = blockIdx.x;
        if (cid >= p.chunk_off[p.B * p.G * p.NSb]) return;
        int lo = 0, hi = p.B * p.G * p.NSb;             // entry e with chunk_off[e] <= cid < chunk_off[e+1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (p.chunk_off[mid] <= cid) lo = mid;
            else hi = mid;
        }
        const int e = lo;
        b = e / (p.G * p.NSb);
        g = (e / p.NSb) % p.G;
        const int j = e % p.NSb;
        const int c = cid - p.chunk_off[e];
        key0 = j * p.lp;
        tok_lo = p.off[e] + c * kBwdChunk;
        tok_hi = min(p.off[e] + p.cnt[e], tok_lo + kBwdChunk);
        toklist = p.list;
    } else if (BR == kBrWin) {
        key0 = blockIdx.x * 64;
        if (key0 >= p.T) return;
        const int tmax = min(p.T, key0 + 64 + p.w - 1);
        tok_lo = key0 + blockIdx.y * kBwdChunk;
        tok_hi = min(tmax, tok_lo + kBwdChunk);
    } else {
        key0 = blockIdx.x * 64;
        if (key0 >= p.C) return;
        const int tfirst = key0 * p.d + p.l - 1;
        tok_lo = tfirst + blockIdx.y * kBwdChunk;
        tok_hi = min(p.T, tok_lo + kBwdChunk);
    }
    if (tok_lo >= tok_hi) return;
    const int nkeys = BR == kBrCmp ? p.C : p.T;

    // the tile's K and V rows (rows past the keys zero-filled)
    {
        const __nv_bfloat16* kb = BR == kBrCmp ? p.kc + ((size_t)b * p.C * p.G + g) * DK
                                               : p.k + ((size_t)b * p.T * p.G + g) * DK;
        const __nv_bfloat16* vb = BR == kBrCmp ? p.vc + ((size_t)b * p.C * p.G + g) * DV
                                               : p.v + ((size_t)b * p.T * p.G + g) * DV;
        const int nv = min(64, nkeys - key0);
        for (int e = threadIdx.x; e < 64 * (DK / 8); e += 128) {
            const int r = e / (DK / 8), c8 = e % (DK / 8);
            const bool ok = r < nv;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(kt + r * KP + c8 * 16)),
                         "l"(kb + (size_t)(ok ? key0 + r : key0) * p.G * DK + c8 * 8), "r"(ok ? 16 : 0)
                         : "memory");
        }
        for (int e = threadIdx.x; e < 64 * (DV / 8); e += 128) {
            const int r = e / (DV / 8), c8 = e % (DV / 8);
            const bool ok = r < nv;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(vt + r * VP + c8 * 16)),
                         "l"(vb + (size_t)(ok ? key0 + r : key0) * p.G * DV + c8 * 8), "r"(ok ? 16 : 0)
                         : "memory");
        }
        cp_async_commit();
    }
    // one token's Q / dO rows (heads past HG zero) and statistics into buffer `buf`
    auto stage = [&](int it, int buf) {
        const int t = toklist ? toklist[it] : it;
        const size_t rowbase = ((size_t)b * p.T + t) * p.H + (size_t)g * p.HG;
        uint8_t* qs = tokb + buf * 16 * (KP + VP);
        uint8_t* ds = qs + 16 * KP;
        for (int e = threadIdx.x; e < 16 * (DK / 8); e += 128) {
            const int h = e / (DK / 8), c8 = e % (DK / 8);
            const bool ok = h < p.HG;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(qs + h * KP + c8 * 16)),
                         "l"(p.q + (rowbase + (ok ? h : 0)) * DK + c8 * 8), "r"(ok ? 16 : 0)
                         : "memory");
        }
        for (int e = threadIdx.x; e < 16 * (DV / 8); e += 128) {
            const int h = e / (DV / 8), c8 = e % (DV / 8);
            const bool ok = h < p.HG;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(ds + h * VP + c8 * 16)),
                         "l"(p.dout + (rowbase + (ok ? h : 0)) * DV + c8 * 8), "r"(ok ? 16 : 0)
                         : "memory");
        }
        cp_async_commit();
        if (threadIdx.x < 16) {
            const int h = threadIdx.x;
            const bool ok = h < p.HG;
            sl[buf][h] = ok ? p.lse2[(rowbase + h) * 3 + BR] : -INFINITY;
            sD[buf][h] = ok ? p.dlt[(rowbase + h) * 3 + BR] : 0.f;
            sg[buf][h] = ok ? p.gates[(rowbase + h) * 3 + BR] : 0.f;
        }
        if (threadIdx.x == 0) stok[buf] = t;
    };

    float dk[DK / 8][4], dv[DV / 8][4];
#pragma unroll
    for (int nt = 0; nt < DK / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) dk[nt][e] = 0.f;
#pragma unroll
    for (int nt = 0; nt < DV / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) dv[nt][e] = 0.f;
    const int mi = lane >> 3, rr = lane & 7;
    const uint32_t ka = smem_u32(kt) + (warp * 16 + (mi & 1) * 8 + rr) * KP + (mi >> 1) * 16;   // A rows of this warp
    const uint32_t va = smem_u32(vt) + (warp * 16 + (mi & 1) * 8 + rr) * VP + (mi >> 1) * 16;
    // key of accumulator rows gr, gr + 8 (tile-local)
    const int kr0 = warp * 16 + gr, kr1 = kr0 + 8;

    stage(tok_lo, 0);
    for (int it = tok_lo; it < tok_hi; ++it) {
        const int buf = (it - tok_lo) & 1;
        if (it + 1 < tok_hi) {
            stage(it + 1, buf ^ 1);
            cp_async_wait_1();
        } else {
            cp_async_wait();
        }
        __syncthreads();
        const int t = stok[buf];
        const uint32_t qs = smem_u32(tokb + buf * 16 * (KP + VP));
        const uint32_t ds = qs + 16 * KP;
        // S^T = K_w Q^T, dP^T = V_w dO^T: two n-tiles of 8 heads
        float sa[2][4], da[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sa[nt][e] = da[nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
            uint32_t a[4], b0, b1, b2, b3;
            ldsm_x4(ka + kk * 32, a[0], a[1], a[2], a[3]);
            // B: heads (mi>>1)*8 + rr, dims kk*16 + (mi&1)*8
            ldsm_x4(qs + ((mi >> 1) * 8 + rr) * KP + kk * 32 + (mi & 1) * 16, b0, b1, b2, b3);
            mma16816(sa[0], a, b0, b1);
            mma16816(sa[1], a, b2, b3);
        }
#pragma unroll
        for (int kk = 0; kk < DV / 16; ++kk) {
            uint32_t a[4], b0, b1, b2, b3;
            ldsm_x4(va + kk * 32, a[0], a[1], a[2], a[3]);
            ldsm_x4(ds + ((mi >> 1) * 8 + rr) * VP + kk * 32 + (mi & 1) * 16, b0, b1, b2, b3);
            mma16816(da[0], a, b0, b1);
            mma16816(da[1], a, b2, b3);
        }
        // which of this thread's two keys does token t see?
        auto seen = [&](int kr) -> bool {
            const int key = key0 + kr;
            if (key >= nkeys) return false;
            if (BR == kBrCmp) return key < ncmp_vis(p, t);
            if (BR == kBrSlc) return key <= t;
            return key <= t && key >= t - p.w + 1;
        };
        const bool v0 = seen(kr0), v1 = seen(kr1);
        float ps[2][4], pg[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int h = nt * 8 + tg * 2 + (e & 1);
                const bool ok = (e < 2 ? v0 : v1) && sl[buf][h] != -INFINITY;
                const float P = ok ? exp2f(sa[nt][e] * p.scale_log2 - sl[buf][h]) : 0.f;
                ps[nt][e] = P * (sg[buf][h] * da[nt][e] - sD[buf][h]);
                pg[nt][e] = P * sg[buf][h];
            }
        // dK_w += dS^T Q, dV_w += (gP)^T dO: A = the 16 x 16 (keys x heads) tile, B from
        // the Q / dO rows (heads = K dimension) via ldmatrix.trans
        uint32_t as[4], ap[4];
        as[0] = pack_bf16x2(ps[0][0], ps[0][1]);
        as[1] = pack_bf16x2(ps[0][2], ps[0][3]);
        as[2] = pack_bf16x2(ps[1][0], ps[1][1]);
        as[3] = pack_bf16x2(ps[1][2], ps[1][3]);
        ap[0] = pack_bf16x2(pg[0][0], pg[0][1]);
        ap[1] = pack_bf16x2(pg[0][2], pg[0][3]);
        ap[2] = pack_bf16x2(pg[1][0], pg[1][1]);
        ap[3] = pack_bf16x2(pg[1][2], pg[1][3]);
#pragma unroll
        for (int nt = 0; nt < DK / 8; nt += 2) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(qs + ((mi & 1) * 8 + rr) * KP + (nt * 8 + (mi >> 1) * 8) * 2, b0, b1, b2, b3);
            mma16816(dk[nt], as, b0, b1);
            mma16816(dk[nt + 1], as, b2, b3);
        }
#pragma unroll
        for (int nt = 0; nt < DV / 8; nt += 2) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(ds + ((mi & 1) * 8 + rr) * VP + (nt * 8 + (mi >> 1) * 8) * 2, b0, b1, b2, b3);
            mma16816(dv[nt], ap, b0, b1);
            mma16816(dv[nt + 1], ap, b2, b3);
        }
        __syncthreads();                        // buffer `buf` is restaged next iteration
    }
    // add into the fp32 outputs (several token chunks share a key tile)
    float* dkb = BR == kBrCmp ? p.dkc + ((size_t)b * p.C * p.G + g) * DK : p.dk + ((size_t)b * p.T * p.G + g) * DK;
    float* dvb = BR == kBrCmp ? p.dvc + ((size_t)b * p.C * p.G + g) * DV : p.dv + ((size_t)b * p.T * p.G + g) * DV;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int key = key0 + (half ? kr1 : kr0);
        if (key >= nkeys) continue;
        float* dkr = dkb + (size_t)key * p.G * DK;
        float* dvr = dvb + (size_t)key * p.G * DV;
#pragma unroll
        for (int nt = 0; nt < DK / 8; ++nt) {
            atomicAdd(dkr + nt * 8 + tg * 2, p.scale * dk[nt][2 * half]);
            atomicAdd(dkr + nt * 8 + tg * 2 + 1, p.scale * dk[nt][2 * half + 1]);
        }
#pragma unroll
        for (int nt = 0; nt < DV / 8; ++nt) {
            atomicAdd(dvr + nt * 8 + tg * 2, dv[nt][2 * half]);
            atomicAdd(dvr + nt * 8 + tg * 2 + 1, dv[nt][2 * half + 1]);
        }
    }
}

// -------------------------------------------------- inverse index (slc)
__global__ void bwd_sel_count(const BwdParams p) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long N = (long long)p.B * p.T * p.G * p.n;
    if (i >= N) return;
    const int j = p.idx[i];
    if (j < 0) return;
    const long long btg = i / p.n;
    const int g = (int)(btg % p.G);
    const int b = (int)(btg / ((long long)p.T * p.G));
    atomicAdd(&p.cnt[((size_t)b * p.G + g) * p.NSb + j], 1);
}

// single CTA of 1024 threads: off = exclusive scan of cnt, chunk_off = scan of ceil(cnt/chunk)
__global__ void __launch_bounds__(1024) bwd_sel_scan(const BwdParams p) {
    __shared__ int s_cnt[1024], s_ch[1024];
    const int N = p.B * p.G * p.NSb;
    const int per = (N + 1023) / 1024;
    const int beg = min(N, (int)threadIdx.x * per), end = min(N, beg + per);
    int a = 0, c = 0;
    for (int i = beg; i < end; ++i) {
        a += p.cnt[i];
        c += (p.cnt[i] + kBwdChunk - 1) / kBwdChunk;
    }
    s_cnt[threadIdx.x] = a;
    s_ch[threadIdx.x] = c;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
        int va = threadIdx.x >= (unsigned)o ? s_cnt[threadIdx.x - o] : 0;
        int vc = threadIdx.x >= (unsigned)o ? s_ch[threadIdx.x - o] : 0;
        __syncthreads();
        s_cnt[threadIdx.x] += va;
        s_ch[threadIdx.x] += vc;
        __syncthreads();
    }
    a = s_cnt[threadIdx.x] - a;
    c = s_ch[threadIdx.x] - c;
    for (int i = beg; i < end; ++i) {
        p.off[i] = a;
        p.chunk_off[i] = c;
        a += p.cnt[i];
        c += (p.cnt[i] + kBwdChunk - 1) / kBwdChunk;
    }
    if (threadIdx.x == 1023) {
        p.off[N] = s_cnt[1023];
        p.chunk_off[N] = s_ch[1023];
    }
}

__global__ void bwd_sel_fill(const BwdParams p) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long N = (long long)p.B * p.T * p.G * p.n;
    if (i >= N) return;
    const int j = p.idx[i];
    if (j < 0) return;
    const long long btg = i / p.n;
    const int g = (int)(btg % p.G);
    const int t = (int)((btg / p.G) % p.T);
    const int b = (int)(btg / ((long long)p.T * p.G));
    const size_t e = ((size_t)b * p.G + g) * p.NSb + j;
    const int pos = atomicAdd(&p.cursor[e], 1);
    p.list[p.off[e] + pos] = t;
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
