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
//   bwd_query_kernel     one CTA per (b, t, g): recomputes every branch's LSE
//                        and o_c, writes dgates and D_c, accumulates dq.
//   bwd_kv_kernel<BR>    key-centric: a tile of 64 keys (raw tokens for the
//                        window and selected branches, compressed blocks for
//                        the compressed one) accumulates over the queries that
//                        read it, then adds into dk/dv (dK~/dV~) atomically.
//                        Selected keys find their queries through an inverse
//                        index (block -> tokens) built by count / scan / fill.
//   bwd_phiT_kernel      dk/dv += phi^T(dK~/dV~).
#pragma once
#include "nsa_dev.cuh"

namespace nsa {

enum { kBrCmp = 0, kBrSlc = 1, kBrWin = 2 };
constexpr int kBwdChunk = 32;      // tokens per key-centric work item

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

// ------------------------------------------------------------ per query
template <int DK, int DV>
__global__ void __launch_bounds__(256) bwd_query_kernel(const BwdParams p) {
    extern __shared__ float sm[];
    float* qf = sm;                                // [16][DK+1]
    float* dof = qf + 16 * (DK + 1);               // [16][DV+1]
    float* Kc = dof + 16 * (DV + 1);               // [64][DK+1]
    float* Vc = Kc + 64 * (DK + 1);                // [64][DV+1]
    float* Sb = Vc + 64 * (DV + 1);                // [16][64]
    float* hl = Sb + 16 * 64;                      // [16] lse2 of the branch
    __shared__ int units[16];
    __shared__ int nunits;
    constexpr int DKT = DK / 16, DVT = DV / 16;

    const int t = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x;
    const size_t rowbase = ((size_t)b * p.T + t) * p.H + (size_t)g * p.HG;
    for (int e = tid; e < 16 * DK; e += 256) {
        const int h = e / DK, c = e % DK;
        qf[h * (DK + 1) + c] = h < p.HG ? __bfloat162float(p.q[(rowbase + h) * DK + c]) : 0.f;
    }
    for (int e = tid; e < 16 * DV; e += 256) {
        const int h = e / DV, c = e % DV;
        dof[h * (DV + 1) + c] = h < p.HG ? __bfloat162float(p.dout[(rowbase + h) * DV + c]) : 0.f;
    }
    if (tid == 0) {
        int nu = 0;
        const int32_t* r = p.idx + (((size_t)b * p.T + t) * p.G + g) * p.n;
        for (int a = 0; a < p.n; ++a)
            if (r[a] >= 0) units[nu++] = r[a];
        nunits = nu;
    }
    __syncthreads();

    const int hq = tid >> 4, cg = tid & 15;        // (head, channel group) layout
    const int kk = tid >> 2, part = tid & 3;       // (key, head quarter) layout
    float dq[DKT];
#pragma unroll
    for (int e = 0; e < DKT; ++e) dq[e] = 0.f;

    for (int br = 0; br < 3; ++br) {
        int nk, lo = 0;
        if (br == kBrCmp) nk = ncmp_vis(p, t);
        else if (br == kBrSlc) nk = nunits * p.lp;
        else {
            lo = max(0, t - p.w + 1);
            nk = t - lo + 1;
        }
        const float gc = p.gates[(rowbase + min(hq, p.HG - 1)) * 3 + br];
        // row pointers of a key of this branch; false for keys the query does not
        // see (tokens after t, which may lie past the end of the sequence)
        auto key_rows = [&](int key, const __nv_bfloat16*& kr, const __nv_bfloat16*& vr) -> bool {
            if (br == kBrCmp) {
                kr = p.kc + (((size_t)b * p.C + key) * p.G + g) * DK;
                vr = p.vc + (((size_t)b * p.C + key) * p.G + g) * DV;
                return true;
            }
            int u = (br == kBrSlc) ? units[key / p.lp] * p.lp + key % p.lp : lo + key;
            kr = p.k + (((size_t)b * p.T + u) * p.G + g) * DK;
            vr = p.v + (((size_t)b * p.T + u) * p.G + g) * DV;
            return u <= t;
        };
        auto load_chunk = [&](int c0) {
            for (int e = tid; e < 64 * DK; e += 256) {
                const int key = e / DK, c = e % DK;
                float val = 0.f;
                if (c0 + key < nk) {
                    const __nv_bfloat16 *kr, *vr;
                    if (key_rows(c0 + key, kr, vr)) val = __bfloat162float(kr[c]);
                }
                Kc[key * (DK + 1) + c] = val;
            }
            for (int e = tid; e < 64 * DV; e += 256) {
                const int key = e / DV, c = e % DV;
                float val = 0.f;
                if (c0 + key < nk) {
                    const __nv_bfloat16 *kr, *vr;
                    if (key_rows(c0 + key, kr, vr)) val = __bfloat162float(vr[c]);
                }
                Vc[key * (DV + 1) + c] = val;
            }
        };
        auto logits = [&](int c0) {
            // thread (key kk, heads part*4 .. part*4+3)
            bool valid = false;
            if (c0 + kk < nk) {
                const __nv_bfloat16 *kr, *vr;
                valid = key_rows(c0 + kk, kr, vr);
            }
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
                const int h = part * 4 + hh;
                float s = 0.f;
                for (int c = 0; c < DK; ++c) s += qf[h * (DK + 1) + c] * Kc[kk * (DK + 1) + c];
                Sb[h * 64 + kk] = valid ? s * p.scale_log2 : -INFINITY;
            }
        };
        // ---- pass 1: LSE and o_c
        float m = -INFINITY, l = 0.f;
        float o[DVT];
#pragma unroll
        for (int e = 0; e < DVT; ++e) o[e] = 0.f;
        for (int c0 = 0; c0 < nk; c0 += 64) {
            load_chunk(c0);
            __syncthreads();
            logits(c0);
            __syncthreads();
            float cm = -INFINITY;
            for (int q2 = cg; q2 < 64; q2 += 16) cm = fmaxf(cm, Sb[hq * 64 + q2]);
#pragma unroll
            for (int s2 = 8; s2 >= 1; s2 >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, s2));
            const float mn = fmaxf(m, cm);
            const float alpha = (mn == -INFINITY) ? 1.f : exp2f(m - mn);
            float ls = 0.f;
            __syncthreads();
            for (int q2 = cg; q2 < 64; q2 += 16) {
                const float sv = Sb[hq * 64 + q2];
                const float e = sv == -INFINITY ? 0.f : exp2f(sv - mn);
                Sb[hq * 64 + q2] = e;
                ls += e;
            }
#pragma unroll
            for (int s2 = 8; s2 >= 1; s2 >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, s2);
            l = l * alpha + ls;
            m = mn;
            __syncthreads();
#pragma unroll
            for (int e = 0; e < DVT; ++e) {
                float acc = 0.f;
                for (int q2 = 0; q2 < 64; ++q2) acc += Sb[hq * 64 + q2] * Vc[q2 * (DV + 1) + cg * DVT + e];
                o[e] = o[e] * alpha + acc;
            }
            __syncthreads();
        }
        float dg = 0.f;
#pragma unroll
        for (int e = 0; e < DVT; ++e) {
            o[e] = l > 0.f ? o[e] / l : 0.f;
            dg += o[e] * dof[hq * (DV + 1) + cg * DVT + e];
        }
#pragma unroll
        for (int s2 = 8; s2 >= 1; s2 >>= 1) dg += __shfl_xor_sync(0xffffffffu, dg, s2);
        const float l2 = l > 0.f ? m + log2f(l) : -INFINITY;
        const float Dc = gc * dg;
        if (cg == 0) {
            hl[hq] = l2;
            if (hq < p.HG) {
                p.dgates[(rowbase + hq) * 3 + br] = dg;
                p.lse2[(rowbase + hq) * 3 + br] = l2;
                p.dlt[(rowbase + hq) * 3 + br] = Dc;
            }
        }
        // D_c of head part*4+hh for the (key, head quarter) layout
        __syncthreads();
        float Dq[4], gq[4];
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
            const int h = part * 4 + hh;
            Dq[hh] = h < p.HG ? p.dlt[(rowbase + h) * 3 + br] : 0.f;
            gq[hh] = h < p.HG ? p.gates[(rowbase + h) * 3 + br] : 0.f;
        }
        // ---- pass 2: dS and dq
        for (int c0 = 0; c0 < nk; c0 += 64) {
            load_chunk(c0);
            __syncthreads();
            logits(c0);
            __syncthreads();
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
                const int h = part * 4 + hh;
                const float sv = Sb[h * 64 + kk];
                const float P = (sv == -INFINITY || hl[h] == -INFINITY) ? 0.f : exp2f(sv - hl[h]);
                float dP = 0.f;
                for (int c = 0; c < DV; ++c) dP += dof[h * (DV + 1) + c] * Vc[kk * (DV + 1) + c];
                dP *= gq[hh];
                Sb[h * 64 + kk] = P * (dP - Dq[hh]);
            }
            __syncthreads();
#pragma unroll
            for (int e = 0; e < DKT; ++e) {
                float acc = 0.f;
                for (int q2 = 0; q2 < 64; ++q2) acc += Sb[hq * 64 + q2] * Kc[q2 * (DK + 1) + cg * DKT + e];
                dq[e] += p.scale * acc;
            }
            __syncthreads();
        }
    }
    if (hq < p.HG) {
#pragma unroll
        for (int e = 0; e < DKT; ++e) p.dq[(rowbase + hq) * DK + cg * DKT + e] = dq[e];
    }
}

// --------------------------------------------------------- per key tile
// grid.z = b*G + g.  WIN: grid (key tiles of 64 tokens, token chunks).
// CMP: grid (key tiles of 64 compressed blocks, token chunks).
// SLC: grid.x = chunk id over the inverse index (binary search), b and g
// from the entry found.
template <int DK, int DV, int BR>
__global__ void __launch_bounds__(256) bwd_kv_kernel(const BwdParams p) {
    __shared__ float qf[16][DK];
    __shared__ float dof[16][DV];
    __shared__ float hl2[16], hD[16];
    constexpr int DK4 = DK / 4, DV4 = DV / 4;
    int b = blockIdx.z / p.G, g = blockIdx.z % p.G;
    const int tid = threadIdx.x, kk = tid >> 2, part = tid & 3;

    int key0, tok_lo, tok_hi;           // keys key0..key0+63; tokens (or list entries) [tok_lo, tok_hi)
    const int* toklist = nullptr;
    if (BR == kBrSlc) {
        const int cid = blockIdx.x;
        if (cid >= p.chunk_off[p.B * p.G * p.NSb]) return;
        // entry e with chunk_off[e] <= cid < chunk_off[e+1]
        int lo = 0, hi = p.B * p.G * p.NSb;
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

    const int key = key0 + kk;
    const int nkeys = BR == kBrCmp ? p.C : p.T;
    const bool key_ok = key < nkeys;
    float kr[DK4], vr[DV4], gk[DK4], gv[DV4];
    {
        const __nv_bfloat16* kp = BR == kBrCmp ? p.kc + (((size_t)b * p.C + key) * p.G + g) * DK
                                               : p.k + (((size_t)b * p.T + key) * p.G + g) * DK;
        const __nv_bfloat16* vp = BR == kBrCmp ? p.vc + (((size_t)b * p.C + key) * p.G + g) * DV
                                               : p.v + (((size_t)b * p.T + key) * p.G + g) * DV;
#pragma unroll
        for (int e = 0; e < DK4; ++e) {
            kr[e] = key_ok ? __bfloat162float(kp[e * 4 + part]) : 0.f;
            gk[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < DV4; ++e) {
            vr[e] = key_ok ? __bfloat162float(vp[e * 4 + part]) : 0.f;
            gv[e] = 0.f;
        }
    }
    for (int it = tok_lo; it < tok_hi; ++it) {
        const int t = toklist ? toklist[it] : it;
        const size_t rowbase = ((size_t)b * p.T + t) * p.H + (size_t)g * p.HG;
        __syncthreads();
        for (int e = tid; e < 16 * DK; e += 256) {
            const int h = e / DK, c = e % DK;
            qf[h][c] = h < p.HG ? __bfloat162float(p.q[(rowbase + h) * DK + c]) : 0.f;
        }
        for (int e = tid; e < 16 * DV; e += 256) {
            const int h = e / DV, c = e % DV;
            dof[h][c] = h < p.HG ? __bfloat162float(p.dout[(rowbase + h) * DV + c]) *
                                       p.gates[(rowbase + h) * 3 + BR]
                                 : 0.f;
        }
        if (tid < 16) {
            hl2[tid] = tid < p.HG ? p.lse2[(rowbase + tid) * 3 + BR] : -INFINITY;
            hD[tid] = tid < p.HG ? p.dlt[(rowbase + tid) * 3 + BR] : 0.f;
        }
        __syncthreads();
        bool valid;
        if (BR == kBrCmp) valid = key_ok && key < ncmp_vis(p, t);
        else if (BR == kBrSlc) valid = key_ok && key <= t;
        else valid = key_ok && key <= t && key >= t - p.w + 1;
        for (int h = 0; h < p.HG; ++h) {
            float s = 0.f, dp = 0.f;
#pragma unroll
            for (int e = 0; e < DK4; ++e) s += qf[h][e * 4 + part] * kr[e];
#pragma unroll
            for (int e = 0; e < DV4; ++e) dp += dof[h][e * 4 + part] * vr[e];
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            dp += __shfl_xor_sync(0xffffffffu, dp, 1);
            dp += __shfl_xor_sync(0xffffffffu, dp, 2);
            const float P = (valid && hl2[h] != -INFINITY) ? exp2f(s * p.scale_log2 - hl2[h]) : 0.f;
            const float dS = P * (dp - hD[h]) * p.scale;
#pragma unroll
            for (int e = 0; e < DK4; ++e) gk[e] += dS * qf[h][e * 4 + part];
#pragma unroll
            for (int e = 0; e < DV4; ++e) gv[e] += P * dof[h][e * 4 + part];
        }
    }
    if (key_ok) {
        float* dkp = BR == kBrCmp ? p.dkc + (((size_t)b * p.C + key) * p.G + g) * DK
                                  : p.dk + (((size_t)b * p.T + key) * p.G + g) * DK;
        float* dvp = BR == kBrCmp ? p.dvc + (((size_t)b * p.C + key) * p.G + g) * DV
                                  : p.dv + (((size_t)b * p.T + key) * p.G + g) * DV;
#pragma unroll
        for (int e = 0; e < DK4; ++e) atomicAdd(dkp + e * 4 + part, gk[e]);
#pragma unroll
        for (int e = 0; e < DV4; ++e) atomicAdd(dvp + e * 4 + part, gv[e]);
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
