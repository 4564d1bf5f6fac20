// k_decode.cuh -- batched decode step (page "硬件对齐+原生训练！DeepSeek NSA打造高效
// 稀疏Attention", 效率分析 解码速度: per step NSA reads the compressed tokens, the
// selected blocks and the window, not the whole cache).
//
// One query per sequence at t = L-1 over packed varlen caches.  The step is
// HBM-bound: every cache row is read once.  The 16 heads of a GQA group are
// the M = 16 side of warp-level bf16 tensor-core products (mma.sync
// m16n8k16, fp32 accumulate).  The two streaming kernels are persistent (one
// CTA of 8 warps per SM).  Each warp pipelines K and V separately (the next
// chunk's K is in flight while this chunk's softmax and P.V run, its V while
// the next logits run) and keeps an online softmax.  Compressed stream: the
// chunks of 32 cache rows of all (seq, group) pairs form one sequence cut into
// equal contiguous ranges, one per warp; a warp streams its range across pair
// boundaries and writes a record per pair it touched at slot (warp index +
// seq*G + group), unique because consecutive pairs share at most one warp.
// Selected/window stream: the same with ranges per CTA, whose warps take a
// pair's chunks round-robin and merge once per pair into one record.
//   1. dec_cmp_stream   compressed cache: per segment (max, sum, unnormalised
//                       O); per chunk the head max and the per-head selection-
//                       block sums of exp(logit - chunk max), mapped with the
//                       overlap weights, so the importance scores can be
//                       normalised exactly once the row LSE is known.
//   2. dec_cmp_combine  per (seq, group): LSE, o_cmp, group importance scores
//                       (sum over heads and chunks of the block sums rescaled
//                       by exp(chunk max - LSE)), top-n by one warp.
//   3. dec_slcwin_stream  the sorted union of the selected blocks and the
//                       window blocks (a fixed number of unit slots per pair,
//                       the unused ones empty): logits once, online softmax of
//                       the selected and the window branch.
//   4. dec_final        merge the records per branch; out = sum_c g_c o_c; lse.
#pragma once
#include "nsa_dev.cuh"
#include "k_topn.cuh"
#include "k_mma.cuh"

namespace nsa {

constexpr int kDecW = 8;             // warps per streaming CTA
constexpr int kDecNBS = 33;          // block-sum slots per chunk (>= (31 + l/d - 1) / (l'/d) + 1)
constexpr int kDecMaxSeqs = 2048;    // sequences per call (chunk prefix held in shared memory)
constexpr int kDecMaxChunks = 256;   // compressed chunks per sequence (T <= 131072, d = 16)
constexpr int kDecMaxUnits = 48;     // units in a (selected U window) list
constexpr int kDecMaxGrid = 1024;    // CTAs of a streaming kernel

struct DecParams {
    int S, H, G, HG, DK, DV;
    int l, d, lp, n, fi, fl, w;
    int spb, cps, nbs;       // l'/d, l/d, block-sum slots used per chunk
    float scale_log2;
    const __nv_bfloat16 *q, *kcache, *vcache, *kccache, *vccache;
    const int64_t *kv_off, *cmp_off;   // row starts; [S+1] packed, or [S] with kv_len
    const int64_t* kv_len;             // [S] tokens per sequence, or null (packed offsets)
    const float* gates;
    float* out;
    int32_t* sel_idx;
    float* lse;
    float* cmax;     // [S*G][NCH][16]            chunk max per head (log2 units)
    float* bsum;     // [S*G][NCH][kDecNBS][16]   per-head block sums of exp2(s - chunk max)
    float* part1;    // [grid1*8 + S*G][16][DV+4] per warp and pair: max, sum, -, -, unnormalised O
    float* lsecmp;   // [S*G][16]                 log2 units
    float* part2;    // [grid3 + S*G][2][16][DV+4] per segment and branch (selected, window)
    int* cpre;       // [S+1] compressed chunks (x G) before sequence s
    int* units;      // [S*G][NUV] selected U window blocks of a pair: block*2 + selected, -1 empty
    int Lmax, Cmax, NCH, NUV, NSmax;
    int grid1, grid3;
};

template <int DK, int DV>
__host__ __device__ constexpr int dec_stage_bytes() {      // one warp: 32 K rows + 32 V rows
    return 32 * ((DK * 2 + 16) + (DV * 2 + 16));
}
template <int DK, int DV>
__host__ __device__ constexpr int dec_stream_smem() {      // staging + P tiles (block sums)
    return kDecW * dec_stage_bytes<DK, DV>() + kDecW * 16 * 33 * 4;
}

// Q of the group's 16 heads (rows >= HG zero) as A fragments for DK/16 k-steps
template <int DK>
__device__ __forceinline__ void load_q_frags(const DecParams& p, int s, int g, uint32_t (&qa)[DK / 16][4]) {
    load_a_frags<DK>(p.q + ((size_t)s * p.H + (size_t)g * p.HG) * DK, p.HG, qa);
}

// lengths of sequence s; false when it is empty or exceeds the sizes the
// workspace was laid out for
__device__ __forceinline__ bool dec_seq_ok(const DecParams& p, int s, int& L, int& C) {
    if (p.kv_len) {               // rows from explicit lengths (caches with spare capacity)
        L = (int)p.kv_len[s];
        C = L >= p.l ? (L - p.l) / p.d + 1 : 0;
    } else {
        L = (int)(p.kv_off[s + 1] - p.kv_off[s]);
        C = (int)(p.cmp_off[s + 1] - p.cmp_off[s]);
    }
    return L > 0 && L <= p.Lmax && C <= p.Cmax;
}

// range of CTA b when N items are cut into `grid` contiguous ranges, and the
// CTA whose range holds item x
__device__ __forceinline__ long long dec_range_start(int b, long long N, int grid) {
    return (long long)b * N / grid;
}
__device__ __forceinline__ int dec_cta_of(long long x, long long N, int grid) {
    return (int)(((x + 1) * grid - 1) / N);
}
// Record slots of items [X0, X1) (X1 > X0): the ranges (warps) that are not
// empty among those holding them, written to out[] (at most cap), found by one
// warp (lane k tests candidate bf + k, 32 at a time); every lane returns the count
__device__ __forceinline__ int dec_record_list_warp(long long X0, long long X1, long long N, int grid, int* out,
                                                    int cap) {
    const int lane = threadIdx.x & 31;
    const int bf = dec_cta_of(X0, N, grid), bl = dec_cta_of(X1 - 1, N, grid);
    int cnt = 0;
    for (int base = bf; base <= bl; base += 32) {
        const int b = base + lane;
        const bool use = b <= bl && dec_range_start(b + 1, N, grid) > dec_range_start(b, N, grid);
        const unsigned m = __ballot_sync(0xffffffffu, use);
        const int pos = cnt + __popc(m & ((1u << lane) - 1u));
        if (use && pos < cap) out[pos] = b;
        cnt += __popc(m);
    }
    return min(cnt, cap);
}

// -------------------------------------------------------------- step 1
template <int DK, int DV>
__global__ void __launch_bounds__(256, 1) dec_cmp_stream(const DecParams p) {
    constexpr int KP = DK * 2 + 16, STG = dec_stage_bytes<DK, DV>();
    extern __shared__ __align__(16) uint8_t dsm[];
    float(*pt)[16][33] = reinterpret_cast<float(*)[16][33]>(dsm + kDecW * STG);  // [8][16][33]
    __shared__ int pre[kDecMaxSeqs + 1];
    __shared__ int64_t cbs[kDecMaxSeqs];             // compressed row start of sequence s
    __shared__ int ccs[kDecMaxSeqs];                 // compressed rows of sequence s
    __shared__ uint64_t kbar[kDecW], vbar[kDecW];    // per warp: its K / V rows landed
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gr = lane >> 2, tg = lane & 3;
    uint8_t* ks = dsm + warp * STG;
    uint8_t* vs = ks + 32 * KP;
    if (threadIdx.x < kDecW) {
        mbar_init(&kbar[threadIdx.x], 1);
        mbar_init(&vbar[threadIdx.x], 1);
    }
    fence_mbar_init();

    // chunks (x G) before sequence s: exclusive prefix by warp 0
    if (warp == 0) {
        int run = 0;
        for (int b0 = 0; b0 < p.S; b0 += 32) {
            const int s = b0 + lane;
            int cnt = 0;
            if (s < p.S) {
                int L, C;
                if (dec_seq_ok(p, s, L, C)) cnt = p.G * ((C + 31) / 32);
                ccs[s] = C;
                cbs[s] = p.cmp_off[s];
            }
            int inc = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += v;
            }
            if (s < p.S) pre[s] = run + inc - cnt;
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) pre[p.S] = run;
    }
    __syncthreads();
    dep_launch();
    if (blockIdx.x == 0)
        for (int s = threadIdx.x; s <= p.S; s += blockDim.x) p.cpre[s] = pre[s];
    const long long N = pre[p.S];
    // Each warp owns a contiguous, equal range of the chunk sequence and streams it
    // on its own: a chunk's K and V copies are issued as soon as the previous
    // chunk has read its staging rows, across (seq, group) boundaries too, and
    // the warp writes one online-softmax record per (seq, group) it touched, at
    // slot (warp index + seq*G + group), unique because consecutive pairs share
    // at most one warp.  No CTA-wide barrier after the prefix.
    const int gw = blockIdx.x * kDecW + warp, W = gridDim.x * kDecW;
    long long x = dec_range_start(gw, N, W);
    const long long x1 = dec_range_start(gw + 1, N, W);
    const float cl = p.scale_log2;
    const bool fast = p.spb == 4 && p.cps == 2;
    uint32_t kph = 0, vph = 0;
    const uint64_t pol = l2_evict_first();
    const size_t kst = (size_t)p.G * DK, vst = (size_t)p.G * DV;
    struct Seg {
        int s, g, c, C, nch;
        int64_t cbase;
    };
    // (seq, group, chunk) of item xx
    auto locate = [&](long long xx, Seg& q) {
        int lo = 0, hi = p.S;                       // largest lo with pre[lo] <= xx
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (pre[mid] <= xx) lo = mid;
            else hi = mid;
        }
        q.s = lo;                                   // lo holds chunks, so it passed the length checks
        q.C = ccs[lo];
        q.nch = (q.C + 31) / 32;
        const int r = (int)(xx - pre[lo]);
        q.g = r / q.nch;
        q.c = r - q.g * q.nch;
        q.cbase = cbs[lo];
    };
    auto issue_k = [&](const Seg& q) {
        warp_bulk_rows<DK>(ks, p.kccache + ((size_t)(q.cbase + (int64_t)q.c * 32) * p.G + q.g) * DK, kst,
                           q.C - q.c * 32, &kbar[warp], pol);
    };
    auto issue_v = [&](const Seg& q) {
        warp_bulk_rows<DV>(vs, p.vccache + ((size_t)(q.cbase + (int64_t)q.c * 32) * p.G + q.g) * DV, vst,
                           q.C - q.c * 32, &vbar[warp], pol);
    };
    if (x < x1) {
        Seg cur;
        locate(x, cur);
        issue_k(cur);
        issue_v(cur);
        uint32_t qa[DK / 16][4];
        load_q_frags<DK>(p, cur.s, cur.g, qa);
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        float o[DV / 8][4];
#pragma unroll
        for (int nt = 0; nt < DV / 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
        for (;;) {
            const int c = cur.c;
            if (!mbar_wait(&kbar[warp], kph, 0x401)) break;   // K of chunk c
            kph ^= 1;
            __syncwarp();
            float sf[4][4];
            warp_logits<DK>(qa, smem_u32(ks), sf);
            __syncwarp();
            // the next item: the following chunk of this pair, or the next pair's first
            const bool more = x + 1 < x1;
            Seg nxt = cur;
            const bool same = c + 1 < cur.nch;
            if (more) {
                if (same) nxt.c = c + 1;
                else locate(x + 1, nxt);
                issue_k(nxt);
            }
            const int nval = min(32, cur.C - c * 32);
            float mc0 = -INFINITY, mc1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = nt * 8 + tg * 2 + (e & 1);
                    const float v = key < nval ? sf[nt][e] * cl : -INFINITY;
                    sf[nt][e] = v;
                    if (e < 2) mc0 = fmaxf(mc0, v);
                    else mc1 = fmaxf(mc1, v);
                }
#pragma unroll
            for (int q2 = 1; q2 <= 2; q2 <<= 1) {
                mc0 = fmaxf(mc0, __shfl_xor_sync(0xffffffffu, mc0, q2));
                mc1 = fmaxf(mc1, __shfl_xor_sync(0xffffffffu, mc1, q2));
            }
            // P relative to the chunk max (key 0 is valid, so the max is finite)
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float pv = exp2f(sf[nt][e] - (e < 2 ? mc0 : mc1));
                    sf[nt][e] = pv;
                    if (e < 2) s0 += pv;
                    else s1 += pv;
                }
#pragma unroll
            for (int q2 = 1; q2 <= 2; q2 <<= 1) {
                s0 += __shfl_xor_sync(0xffffffffu, s0, q2);
                s1 += __shfl_xor_sync(0xffffffffu, s1, q2);
            }
            // per-head selection-block sums of this chunk: slot jl = block 32c/spb + jl
            // takes chunk key i with weight |[i, i+cps) n [jl*spb, jl*spb+spb)|
            const size_t cr = ((size_t)cur.s * p.G + cur.g) * p.NCH + c;
            float* bdst = p.bsum + cr * kDecNBS * 16;
            if (fast) {
                // spb = 4, cps = 2: slot jl = 2 A_jl - P(4jl+3) + P(4jl-1), A = sum of the
                // block's 4 keys; slot 8 = P(31).  Lane pair (tg 0,1) holds block 2nt,
                // pair (2,3) block 2nt+1 of n-tile nt.
#pragma unroll
                for (int rh = 0; rh < 2; ++rh) {
                    float prev3 = 0.f;
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt) {
                        const float x0 = sf[nt][2 * rh], x1v = sf[nt][2 * rh + 1];
                        const float ps = x0 + x1v;
                        const float A = ps + __shfl_xor_sync(0xffffffffu, ps, 1);
                        const float last = __shfl_sync(0xffffffffu, x1v, lane | 1);
                        const float l1q = __shfl_sync(0xffffffffu, x1v, (lane & ~3) | 1);
                        const float l3q = __shfl_sync(0xffffffffu, x1v, (lane & ~3) | 3);
                        const float prev = (tg >> 1) ? l1q : prev3;
                        const float v = 2.f * A - last + prev;
                        if ((tg & 1) == 0 && gr + 8 * rh < p.HG)
                            bdst[(2 * nt + (tg >> 1)) * 16 + gr + 8 * rh] = v;
                        prev3 = l3q;
                    }
                    if (tg == 0 && gr + 8 * rh < p.HG) bdst[8 * 16 + gr + 8 * rh] = prev3;
                }
            } else {
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) pt[warp][e < 2 ? gr : gr + 8][nt * 8 + tg * 2 + (e & 1)] = sf[nt][e];
                __syncwarp();
                if (lane < p.nbs) {
                    const int jk0 = lane * p.spb;
                    const int ilo = max(0, jk0 - p.cps + 1), ihi = min(32, jk0 + p.spb);
                    for (int rr = 0; rr < p.HG; ++rr) {
                        float a = 0.f;
                        for (int k2 = ilo; k2 < ihi; ++k2)
                            a += (float)(min(k2 + p.cps, jk0 + p.spb) - max(k2, jk0)) * pt[warp][rr][k2];
                        bdst[lane * 16 + rr] = a;
                    }
                }
                __syncwarp();
            }
            if (tg == 0) {
                p.cmax[cr * 16 + gr] = mc0;
                p.cmax[cr * 16 + gr + 8] = mc1;
            }
            if (!mbar_wait(&vbar[warp], vph, 0x402)) break;   // V of chunk c
            vph ^= 1;
            __syncwarp();
            // online softmax for O: rescale to the new running max
            const float mn0 = fmaxf(m0, mc0), mn1 = fmaxf(m1, mc1);
            const float a0 = exp2f(m0 - mn0), a1 = exp2f(m1 - mn1);
            const float f0 = exp2f(mc0 - mn0), f1 = exp2f(mc1 - mn1);
            m0 = mn0;
            m1 = mn1;
            l0 = l0 * a0 + s0 * f0;
            l1 = l1 * a1 + s1 * f1;
#pragma unroll
            for (int nt = 0; nt < DV / 8; ++nt) {
                o[nt][0] *= a0;
                o[nt][1] *= a0;
                o[nt][2] *= a1;
                o[nt][3] *= a1;
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                sf[nt][0] *= f0;
                sf[nt][1] *= f0;
                sf[nt][2] *= f1;
                sf[nt][3] *= f1;
            }
            warp_pv<DV>(sf, smem_u32(vs), o);
            __syncwarp();
            if (more) issue_v(nxt);
            if (!more || !same) {
                // this warp's record of (seq, group): (max, sum, -, -, O relative to max)
                constexpr int REC = DV + 4;
                const size_t sg = (size_t)cur.s * p.G + cur.g;
                float* rec = p.part1 + ((size_t)gw + sg) * 16 * REC;
                if (tg == 0) {
                    rec[gr * REC] = m0;
                    rec[gr * REC + 1] = l0;
                    rec[(gr + 8) * REC] = m1;
                    rec[(gr + 8) * REC + 1] = l1;
                }
#pragma unroll
                for (int nt = 0; nt < DV / 8; ++nt) {
                    const int cc = 4 + nt * 8 + tg * 2;
                    *reinterpret_cast<float2*>(rec + gr * REC + cc) = make_float2(o[nt][0], o[nt][1]);
                    *reinterpret_cast<float2*>(rec + (gr + 8) * REC + cc) = make_float2(o[nt][2], o[nt][3]);
                }
                m0 = m1 = -INFINITY;
                l0 = l1 = 0.f;
#pragma unroll
                for (int nt = 0; nt < DV / 8; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
                if (more) load_q_frags<DK>(p, nxt.s, nxt.g, qa);
            }
            if (!more) break;
            cur = nxt;
            ++x;
        }
    }
}

// sorted union of the selected blocks (sel: n entries, -1 padded, ascending)
// and the blocks overlapping the window; flag[i] = 1 when list[i] is selected
__device__ __forceinline__ int dec_units(const DecParams& p, const int32_t* sel, int L, int* list, int* flag) {
    const int wlo = max(0, L - p.w) / p.lp, whi = (L - 1) / p.lp;
    int i = 0, j = wlo, cnt = 0, last = -1;
    while (cnt < kDecMaxUnits) {
        const int a = (i < p.n && sel[i] >= 0) ? sel[i] : 0x7fffffff;
        const int b = j <= whi ? j : 0x7fffffff;
        const int m = min(a, b);
        if (m == 0x7fffffff) break;
        const bool from_sel = m == a;
        if (m == a) ++i;
        if (m == b) ++j;
        if (m != last) {
            list[cnt] = m;
            flag[cnt] = from_sel ? 1 : 0;
            ++cnt;
        } else if (from_sel) {
            flag[cnt - 1] = 1;
        }
        last = m;
    }
    return cnt;
}

// dec_units by one warp, written as units[i] = block*2 + selected (-1 past the
// end, NUV slots): lane i holds selected block i, lane k window block wlo + k;
// a block's place is the number of list entries below it.
// scratch: >= 32 + 2 * kDecMaxUnits ints of shared memory (the one-lane path).
__device__ __forceinline__ void dec_units_warp(const DecParams& p, const int32_t* sel, int L, int* units,
                                               int* scratch) {
    const int lane = threadIdx.x & 31;
    const int wlo = max(0, L - p.w) / p.lp, whi = (L - 1) / p.lp, nw = whi - wlo + 1;
    if (nw > 32) {                                     // windows of more than 32 blocks: one lane
        if (lane == 0) {
            int* sb = scratch;
            int* list = scratch + 32;
            int* flag = scratch + 32 + kDecMaxUnits;
            for (int i = 0; i < p.n; ++i) sb[i] = sel[i];
            const int cnt = dec_units(p, sb, L, list, flag);
            for (int i = 0; i < p.NUV; ++i) units[i] = i < cnt ? list[i] * 2 + flag[i] : -1;
        }
        return;
    }
    const int a = lane < p.n ? sel[lane] : -1;        // ascending, -1 padded
    const bool va = a >= 0;
    const bool inw = va && a >= wlo && a <= whi;
    const bool out = va && !inw;
    const unsigned mout = __ballot_sync(0xffffffffu, out);
    const unsigned mbelow = __ballot_sync(0xffffffffu, out && a < wlo);
    const unsigned selw = __reduce_or_sync(0xffffffffu, inw ? 1u << (a - wlo) : 0u);   // window blocks selected
    const unsigned lt = (1u << lane) - 1u;
    if (out) units[__popc(mout & lt) + (a > whi ? nw : 0)] = a * 2 + 1;
    if (lane < nw) units[lane + __popc(mbelow)] = (wlo + lane) * 2 + ((selw >> lane) & 1u);
    const int cnt = nw + __popc(mout);
    for (int i = cnt + lane; i < p.NUV; i += 32) units[i] = -1;
}

// -------------------------------------------------------------- step 2
// Every load that does not need the row LSE (chunk maxima, this thread's block
// sums) is issued before the first barrier; the records give the LSE in one
// round of loads (their O is merged by the final step); the top-n and the unit
// list run on all warps.
template <int DV>
__global__ void __launch_bounds__(256) dec_cmp_combine(const DecParams p) {
    constexpr int REC = DV + 4;
    extern __shared__ float csm[];                     // fac [NCH][16], pg [NSmax]
    __shared__ int recb[kDecMaxChunks];
    __shared__ int nrec;
    __shared__ int tsm[2 * 8 * 32];                   // top-n scratch
    const int g = blockIdx.x, s = blockIdx.y;
    dep_launch();
    int L, C;
    if (!dec_seq_ok(p, s, L, C)) {
        if (threadIdx.x == 0 && g == 0 && L > 0) atomicOr(&g_nsa_error, 4u);
        return;
    }
    const int t = L - 1;
    const int nch = (C + 31) / 32;
    const size_t sg = (size_t)s * p.G + g;
    dep_wait();                                        // the compressed stream's records
    if (threadIdx.x < 32) {
        int cnt = 0;
        if (nch > 0) {
            const long long X0 = (long long)p.cpre[s] + (long long)g * nch;
            cnt = dec_record_list_warp(X0, X0 + nch, p.cpre[p.S], p.grid1 * kDecW, recb, kDecMaxChunks);
        }
        if (threadIdx.x == 0) nrec = cnt;
    }
    // When no warp range is empty (at least as many chunks as warps), the pair's records
    // are those of the consecutive warps bf .. bl: the LSE's record loads (this
    // thread's first four) are issued now, before the list is shared.
    const int hh = threadIdx.x >> 4, hsub = threadIdx.x & 15;
    float rm0[4], rl0[4];
    int nr_direct = -1;
    {
        const long long NN = p.cpre[p.S];
        const int W1 = p.grid1 * kDecW;
        if (nch > 0 && NN >= W1) {
            const long long X0 = (long long)p.cpre[s] + (long long)g * nch;
            const int bf = dec_cta_of(X0, NN, W1);
            nr_direct = dec_cta_of(X0 + nch - 1, NN, W1) - bf + 1;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = hsub + 16 * k;
                const float* r = p.part1 + ((size_t)(bf + (i < nr_direct ? i : 0)) + sg) * 16 * REC + (size_t)hh * REC;
                rm0[k] = i < nr_direct ? r[0] : -INFINITY;
                rl0[k] = i < nr_direct ? r[1] : 0.f;
            }
        }
    }
    float* fac = csm;
    float* pg = fac + p.NCH * 16;
    // chunk maxima (log2 units) and this thread's block sums: independent of the LSE
    const float* cm = p.cmax + sg * p.NCH * 16;
    for (int e = threadIdx.x; e < nch * 16; e += blockDim.x) fac[e] = cm[e];
    const int NSs = t / p.lp + 1;
    const int bpc = 32 / p.spb;                        // blocks starting in one chunk
    const float* bs = p.bsum + sg * p.NCH * kDecNBS * 16;
    // block j takes the chunks holding keys j*spb-cps+1 .. j*spb+spb-1 (at most two)
    auto block_chunks = [&](int j, int& ca, int& cb) {
        const int ilo = max(0, j * p.spb - p.cps + 1), ihi = min(C - 1, j * p.spb + p.spb - 1);
        ca = ilo >> 5;
        cb = ilo <= ihi ? (ihi >> 5) : ca - 1;
    };
    float4 bv[4][2][4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int j = threadIdx.x + q * blockDim.x;
        int ca, cb;
        block_chunks(j, ca, cb);
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
            const int cc = ca + qq, jl = j - cc * bpc;
            const bool use = j < NSs && cc <= cb && jl >= 0 && jl < p.nbs;
            const float4* bp = reinterpret_cast<const float4*>(bs + ((size_t)(use ? cc : 0) * kDecNBS + (use ? jl : 0)) * 16);
#pragma unroll
            for (int h4 = 0; h4 < 4; ++h4)
                bv[q][qq][h4] = (use && h4 * 4 < p.HG) ? bp[h4] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    __syncthreads();                                   // nrec, recb, fac (raw)
    const int nr = nrec;
    {   // LSE per head over the records: 16 threads per head, each thread's records
        // (i = sub, sub + 16, ...) read once, up to four at a time
        const int h = hh, sub = hsub;
        float M = -INFINITY, Ls = 0.f;
        for (int i0 = sub; i0 < nr; i0 += 64) {
            float rm[4], rl[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = i0 + 16 * k;
                if (i0 == sub && nr_direct >= 0) {      // loaded before the barrier
                    rm[k] = rm0[k];
                    rl[k] = rl0[k];
                } else {
                    const float* r = p.part1 + ((size_t)(recb[i < nr ? i : 0] + sg) * 16 + h) * REC;
                    rm[k] = i < nr ? r[0] : -INFINITY;
                    rl[k] = i < nr ? r[1] : 0.f;
                }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (rm[k] == -INFINITY) continue;
                const float Mn = fmaxf(M, rm[k]);
                Ls = Ls * exp2f(M - Mn) + rl[k] * exp2f(rm[k] - Mn);      // M = -inf first: factor 0
                M = Mn;
            }
        }
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) {
            const float Mo = __shfl_xor_sync(0xffffffffu, M, o), Lo = __shfl_xor_sync(0xffffffffu, Ls, o);
            const float Mn = fmaxf(M, Mo);
            Ls = (Mn == -INFINITY) ? 0.f : Ls * exp2f(M - Mn) + Lo * exp2f(Mo - Mn);
            M = Mn;
        }
        const float l2 = Ls > 0.f ? M + log2f(Ls) : -INFINITY;
        if (sub == 0) p.lsecmp[sg * 16 + h] = l2;
        // per chunk of this head: exp2(chunk max - LSE); heads past HG do not score
        for (int c = sub; c < nch; c += 16)
            fac[c * 16 + h] = (h < p.HG && l2 != -INFINITY) ? exp2f(fac[c * 16 + h] - l2) : 0.f;
    }
    __syncthreads();
    auto dot16 = [&](const float4 (&v)[4], const float* f) {
        float acc = 0.f;
#pragma unroll
        for (int h4 = 0; h4 < 4; ++h4)
            acc += v[h4].x * f[h4 * 4] + v[h4].y * f[h4 * 4 + 1] + v[h4].z * f[h4 * 4 + 2] + v[h4].w * f[h4 * 4 + 3];
        return acc;
    };
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int j = threadIdx.x + q * blockDim.x;
        if (j < NSs) {
            int ca, cb;
            block_chunks(j, ca, cb);
            float acc = 0.f;
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
                const int cc = ca + qq, jl = j - cc * bpc;
                if (cc <= cb && jl >= 0 && jl < p.nbs) acc += dot16(bv[q][qq], fac + cc * 16);
            }
            pg[j] = acc;
        }
    }
    for (int j = threadIdx.x + 4 * blockDim.x; j < NSs; j += blockDim.x) {   // rows longer than 1024 blocks
        int ca, cb;
        block_chunks(j, ca, cb);
        float acc = 0.f;
        for (int cc = ca; cc <= cb; ++cc) {
            const int jl = j - cc * bpc;
            if (jl < 0 || jl >= p.nbs) continue;
            const float* bp = bs + ((size_t)cc * kDecNBS + jl) * 16;
            for (int h = 0; h < p.HG; ++h) acc += bp[h] * fac[cc * 16 + h];
        }
        pg[j] = acc;
    }
    __syncthreads();
    topn_row_cta_redux<256>(pg, t, p.n, p.lp, p.fi, p.fl, p.sel_idx + sg * p.n, tsm);
    // the pair's units for the selected/window stream: the sorted union of the
    // selected blocks and the window's blocks, each flagged when selected
    __syncthreads();                                   // the selection row is written
    if (threadIdx.x < 32) dec_units_warp(p, p.sel_idx + sg * p.n, L, p.units + sg * p.NUV, tsm);
}

// -------------------------------------------------------------- step 3
template <int DK, int DV>
__host__ __device__ constexpr int dec_slcwin_smem() {        // staging + one Q tile per warp
    return kDecW * dec_stage_bytes<DK, DV>() + kDecW * 16 * (DK * 2 + 16);
}

// Each warp owns a contiguous, equal range of the unit slots (NUV per pair, the
// combine's sorted union of selected and window blocks, -1 when empty); per pair
// it loads its own copy of Q and streams the chunks of the pair's units in its
// range, then writes one record per branch at slot (warp index + seq*G + group),
// unique because consecutive pairs share at most one warp.
template <int DK, int DV>
__global__ void __launch_bounds__(256, 1) dec_slcwin_stream(const DecParams p) {
    constexpr int KP = DK * 2 + 16, STG = dec_stage_bytes<DK, DV>();
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ uint64_t kbar[kDecW], vbar[kDecW];
    __shared__ int ulw[kDecW][33];                    // per warp: a batch's non-empty units, their count
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tg = lane & 3;
    uint8_t* ks = dsm + warp * STG;
    uint8_t* vs = ks + 32 * KP;
    uint8_t* qs = dsm + kDecW * STG + warp * 16 * KP;   // this warp's [16][DK] Q tile
    if (threadIdx.x < kDecW) {
        mbar_init(&kbar[threadIdx.x], 1);
        mbar_init(&vbar[threadIdx.x], 1);
    }
    fence_mbar_init();
    __syncthreads();
    dep_launch();
    dep_wait();                                       // the combine's units and selections
    uint32_t kph = 0, vph = 0;
    const uint64_t pol = l2_evict_first();
    const long long U = (long long)p.S * p.G * p.NUV;
    const int gw = blockIdx.x * kDecW + warp, W = gridDim.x * kDecW;
    long long x = dec_range_start(gw, U, W);
    const long long x1 = dec_range_start(gw + 1, U, W);
    const float cl = p.scale_log2;
    constexpr int REC = DV + 4;
    while (x < x1) {
        const size_t sg = (size_t)(x / p.NUV);
        const int ua = (int)(x % p.NUV);
        const int nslot = (int)min((long long)(p.NUV - ua), x1 - x);
        const int s = (int)(sg / p.G), g = (int)(sg % p.G);
        int L, C;
        const bool ok = dec_seq_ok(p, s, L, C);
        const int64_t kvb = ok ? p.kv_off[s] : 0;
        const size_t kst = (size_t)p.G * DK, vst = (size_t)p.G * DV;

        auto tok0 = [&](int u, int i) { return (u >> 1) * p.lp + (i & 1) * 32; };
        // rows past the cache are not read; the source stays inside the sequence
        auto issue_k = [&](int u0) {
            const int nv = min(32, L - u0);
            warp_bulk_rows<DK>(ks, p.kcache + ((size_t)(kvb + (nv > 0 ? u0 : 0)) * p.G + g) * DK, kst, nv, &kbar[warp], pol);
        };
        auto issue_v = [&](int u0) {
            const int nv = min(32, L - u0);
            warp_bulk_rows<DV>(vs, p.vcache + ((size_t)(kvb + (nv > 0 ? u0 : 0)) * p.G + g) * DV, vst, nv, &vbar[warp], pol);
        };
        float m[2][2], l[2][2];
        float o[2][DV / 8][4];
#pragma unroll
        for (int br = 0; br < 2; ++br) {
            m[br][0] = m[br][1] = -INFINITY;
            l[br][0] = l[br][1] = 0.f;
#pragma unroll
            for (int nt = 0; nt < DV / 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) o[br][nt][e] = 0.f;
        }
        const int wlo = L - p.w;
        bool live = true, qready = false;
        // this range's units of the pair, 32 slots at a time (lane i: slot ua + b0 + i)
        for (int b0 = 0; b0 < nslot && live; b0 += 32) {
        {
            const int myu = (ok && b0 + lane < nslot) ? p.units[sg * p.NUV + ua + b0 + lane] : -1;
            const unsigned umask = __ballot_sync(0xffffffffu, myu >= 0);
            if (myu >= 0) ulw[warp][__popc(umask & ((1u << lane) - 1u))] = myu;
            if (lane == 0) ulw[warp][32] = __popc(umask);
        }
        __syncwarp();
        const int n = 2 * ulw[warp][32];                   // chunks of 32 tokens
        // unit of chunk i: the (i/2)-th non-empty slot of the batch
        auto unit_of = [&](int i) { return ulw[warp][i >> 1]; };
        int ucur = n > 0 ? unit_of(0) : 0;
        if (n > 0) {
            issue_k(tok0(ucur, 0));
            issue_v(tok0(ucur, 0));
            if (!qready) {
                // Q of the group as a [16][DK] tile (rows >= HG zero), read with ldmatrix;
                // loaded while the first rows are in flight
                for (int e = lane; e < 16 * (DK / 8); e += 32) {
                    const int h = e / (DK / 8), c8 = e % (DK / 8);
                    int4 v = make_int4(0, 0, 0, 0);
                    if (h < p.HG)
                        v = *reinterpret_cast<const int4*>(p.q + ((size_t)s * p.H + (size_t)g * p.HG + h) * DK + c8 * 8);
                    *reinterpret_cast<int4*>(qs + h * KP + c8 * 16) = v;
                }
                __syncwarp();
                qready = true;
            }
        }
        for (int i = 0; i < n; ++i) {
            const bool more = i + 1 < n;
            const int unxt = more ? ((i & 1) ? unit_of(i + 1) : ucur) : ucur;
            const int u0 = tok0(ucur, i);
            const bool insel = (ucur & 1) != 0;
            const int nval = min(32, L - u0);
            // warp-uniform: does the chunk hold keys of each branch?
            const bool has_sel = insel && nval > 0;
            const bool has_win = nval > 0 && u0 + nval - 1 >= wlo;
            if (!mbar_wait(&kbar[warp], kph, 0x403)) {   // K of chunk i
                live = false;
                break;
            }
            kph ^= 1;
            __syncwarp();
            float sf[4][4];
            if (has_sel || has_win) warp_logits_sa<DK>(smem_u32(qs), smem_u32(ks), sf);
            __syncwarp();
            if (more) issue_k(tok0(unxt, i + 1));
            if (!mbar_wait(&vbar[warp], vph, 0x404)) {   // V of chunk i
                live = false;
                break;
            }
            vph ^= 1;
            __syncwarp();
#pragma unroll
            for (int br = 0; br < 2; ++br) {
                if (br == 0 ? !has_sel : !has_win) continue;
                float pf4[4][4];
                float mc0 = -INFINITY, mc1 = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int key = nt * 8 + tg * 2 + (e & 1);
                        const bool okk = key < nval && (br == 0 || u0 + key >= wlo);
                        const float v = okk ? sf[nt][e] * cl : -INFINITY;
                        pf4[nt][e] = v;
                        if (e < 2) mc0 = fmaxf(mc0, v);
                        else mc1 = fmaxf(mc1, v);
                    }
#pragma unroll
                for (int q2 = 1; q2 <= 2; q2 <<= 1) {
                    mc0 = fmaxf(mc0, __shfl_xor_sync(0xffffffffu, mc0, q2));
                    mc1 = fmaxf(mc1, __shfl_xor_sync(0xffffffffu, mc1, q2));
                }
                const float mn0 = fmaxf(m[br][0], mc0), mn1 = fmaxf(m[br][1], mc1);
                float s0 = 0.f, s1 = 0.f;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float v = pf4[nt][e];
                        const float pv = v == -INFINITY ? 0.f : exp2f(v - (e < 2 ? mn0 : mn1));
                        pf4[nt][e] = pv;
                        if (e < 2) s0 += pv;
                        else s1 += pv;
                    }
#pragma unroll
                for (int q2 = 1; q2 <= 2; q2 <<= 1) {
                    s0 += __shfl_xor_sync(0xffffffffu, s0, q2);
                    s1 += __shfl_xor_sync(0xffffffffu, s1, q2);
                }
                const float a0 = mn0 == -INFINITY ? 1.f : exp2f(m[br][0] - mn0);
                const float a1 = mn1 == -INFINITY ? 1.f : exp2f(m[br][1] - mn1);
                m[br][0] = mn0;
                m[br][1] = mn1;
                l[br][0] = l[br][0] * a0 + s0;
                l[br][1] = l[br][1] * a1 + s1;
#pragma unroll
                for (int nt = 0; nt < DV / 8; ++nt) {
                    o[br][nt][0] *= a0;
                    o[br][nt][1] *= a0;
                    o[br][nt][2] *= a1;
                    o[br][nt][3] *= a1;
                }
                warp_pv<DV>(pf4, smem_u32(vs), o[br]);
            }
            __syncwarp();
            if (more) issue_v(tok0(unxt, i + 1));
            ucur = unxt;
        }
        }
        if (!live) break;
        // this warp's records of the pair, one per branch: (max, sum, -, -, O relative to max)
        float* rec = p.part2 + ((size_t)gw + sg) * 2 * 16 * REC;
        const int gr = lane >> 2;
#pragma unroll
        for (int br = 0; br < 2; ++br) {
            float* rb = rec + br * 16 * REC;
            if (tg == 0) {
                rb[gr * REC] = m[br][0];
                rb[gr * REC + 1] = l[br][0];
                rb[(gr + 8) * REC] = m[br][1];
                rb[(gr + 8) * REC + 1] = l[br][1];
            }
#pragma unroll
            for (int nt = 0; nt < DV / 8; ++nt) {
                const int cc = 4 + nt * 8 + tg * 2;
                *reinterpret_cast<float2*>(rb + gr * REC + cc) = make_float2(o[br][nt][0], o[br][nt][1]);
                *reinterpret_cast<float2*>(rb + (gr + 8) * REC + cc) = make_float2(o[br][nt][2], o[br][nt][3]);
            }
        }
        __syncwarp();                                  // the Q tile is reloaded for the next pair
        x += nslot;
    }
}

// -------------------------------------------------------------- step 4
// Per (seq, group) and eight heads (grid z): the records of all three
// branches merged in two rounds of loads, each round issued at once.  Round 1:
// warp w takes the compressed records of head w (weight exp2(m - LSE) under
// the combine's LSE) and the selected/window records of two (branch, head)
// groups, 16 lanes per group (the branch max M, sum L and the weight
// exp2(m - M) / L of every record).  Round 2: one thread per output float4
// (two for d_v = 64, each taking every other record) sums the weighted O of
// the records, eight of each kind per batch of loads; then
// out = sum_c g_c o_c and the LSEs.  256 CTAs of at most 128 registers per
// thread fit the GPU in one wave.
constexpr int kDecFinalHeads = 8;      // heads per dec_final CTA

template <int DV>
__global__ void __launch_bounds__(256, 2) dec_final(const DecParams p) {
    constexpr int REC = DV + 4, HQ = kDecFinalHeads, NOUT = HQ * DV / 4, NHALF = 256 / NOUT;
    static_assert(NHALF >= 1 && NHALF <= 2 && NHALF * NOUT == 256, "threads per output float4");
    __shared__ int recb[kDecMaxUnits];
    __shared__ int recc[kDecMaxChunks];
    __shared__ int nrec, nrecc;
    __shared__ float wgt[kDecMaxUnits][2][HQ];      // selected/window record weight per branch and head
    __shared__ float wgc[kDecMaxChunks][HQ];        // compressed record weight per head
    __shared__ float lsb[2][HQ];                    // branch LSE (log2 units)
    __shared__ float4 part[NHALF > 1 ? NOUT : 1][3];   // the second thread's sums per output
    const int g = blockIdx.x, s = blockIdx.y, h0 = blockIdx.z * HQ;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int L, C;
    if (h0 >= p.HG || !dec_seq_ok(p, s, L, C)) return;
    const size_t sg = (size_t)s * p.G + g;
    const int nch = (C + 31) / 32;
    dep_wait();                                       // the selected/window records
    if (warp == 0) {
        const long long X0 = (long long)sg * p.NUV;
        const int cnt = dec_record_list_warp(X0, X0 + p.NUV, (long long)p.S * p.G * p.NUV, p.grid3 * kDecW, recb,
                                             kDecMaxUnits);
        if (lane == 0) nrec = cnt;
    } else if (warp == 1) {
        int cnt = 0;
        if (nch > 0) {
            const long long X0 = (long long)p.cpre[s] + (long long)g * nch;
            cnt = dec_record_list_warp(X0, X0 + nch, p.cpre[p.S], p.grid1 * kDecW, recc, kDecMaxChunks);
        }
        if (lane == 0) nrecc = cnt;
    }
    __syncthreads();
    const int nr = nrec, nrc = nrecc;
    {
        // compressed records of head h0 + warp (lane: records lane, lane + 32, ...) and
        // selected/window records of group (branch, head) gi (16 lanes), loads first
        const int hc = h0 + warp;
        const float lc = hc < p.HG ? p.lsecmp[sg * 16 + hc] : -INFINITY;
        const int gi = warp * 2 + (lane >> 4), sub = lane & 15;
        const int br = gi / HQ, hl = gi % HQ, h = h0 + hl;
        constexpr int PC = kDecMaxChunks / 32, PR = (kDecMaxUnits + 15) / 16;
        float cm[PC], rm[PR], rl[PR];
#pragma unroll
        for (int k = 0; k < PC; ++k) {
            const int i = lane + 32 * k;
            cm[k] = (i < nrc && lc != -INFINITY) ? p.part1[((size_t)(recc[i] + sg) * 16 + hc) * REC] : -INFINITY;
        }
#pragma unroll
        for (int k = 0; k < PR; ++k) {
            const int i = sub + 16 * k;
            const bool use = i < nr && h < p.HG;
            const float* r = p.part2 + ((((size_t)recb[use ? i : 0] + sg) * 2 + br) * 16 + (use ? h : 0)) * REC;
            rm[k] = use ? r[0] : -INFINITY;
            rl[k] = use ? r[1] : 0.f;
        }
#pragma unroll
        for (int k = 0; k < PC; ++k) {
            const int i = lane + 32 * k;
            if (i < nrc) wgc[i][warp] = cm[k] != -INFINITY ? exp2f(cm[k] - lc) : 0.f;
        }
        float M = -INFINITY;
#pragma unroll
        for (int k = 0; k < PR; ++k) M = fmaxf(M, rm[k]);
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float Ls = 0.f;
#pragma unroll
        for (int k = 0; k < PR; ++k)
            if (rm[k] != -INFINITY) Ls += rl[k] * exp2f(rm[k] - M);
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
        const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
#pragma unroll
        for (int k = 0; k < PR; ++k) {
            const int i = sub + 16 * k;
            if (i < nr) wgt[i][br][hl] = rm[k] == -INFINITY ? 0.f : exp2f(rm[k] - M) * inv;
        }
        if (sub == 0) lsb[br][hl] = Ls > 0.f ? M + log2f(Ls) : -INFINITY;
    }
    __syncthreads();
    // round 2: output e (head h0 + e / (DV/4), channels c4 .. c4+3)
    const int e = threadIdx.x % NOUT, half = threadIdx.x / NOUT;
    const int hl = e / (DV / 4), c4 = (e % (DV / 4)) * 4, h = h0 + hl;
    const bool active = h < p.HG;
    float4 acc[3];
#pragma unroll
    for (int q = 0; q < 3; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    auto fma4 = [](float4& a, const float4& v, float w) {
        a.x = fmaf(v.x, w, a.x);
        a.y = fmaf(v.y, w, a.y);
        a.z = fmaf(v.z, w, a.z);
        a.w = fmaf(v.w, w, a.w);
    };
    const int nmax = max(nr, nrc);
    for (int i0 = half; active && i0 < nmax; i0 += 8 * NHALF) {
        float4 vc[8], vs[8], vw[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int i = i0 + NHALF * k;
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            vc[k] = (i < nrc && wgc[i][hl] != 0.f)
                        ? *reinterpret_cast<const float4*>(p.part1 + ((size_t)(recc[i] + sg) * 16 + h) * REC + 4 + c4)
                        : z;
            vs[k] = (i < nr && wgt[i][0][hl] != 0.f)
                        ? *reinterpret_cast<const float4*>(p.part2 + ((((size_t)recb[i] + sg) * 2 + 0) * 16 + h) * REC + 4 + c4)
                        : z;
            vw[k] = (i < nr && wgt[i][1][hl] != 0.f)
                        ? *reinterpret_cast<const float4*>(p.part2 + ((((size_t)recb[i] + sg) * 2 + 1) * 16 + h) * REC + 4 + c4)
                        : z;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int i = i0 + NHALF * k;
            fma4(acc[0], vc[k], i < nrc ? wgc[i][hl] : 0.f);
            fma4(acc[1], vs[k], i < nr ? wgt[i][0][hl] : 0.f);
            fma4(acc[2], vw[k], i < nr ? wgt[i][1][hl] : 0.f);
        }
    }
    if (NHALF > 1) {
        if (half == 1) {
#pragma unroll
            for (int q = 0; q < 3; ++q) part[e][q] = acc[q];
        }
        __syncthreads();
    }
    if (half == 0 && active) {
        if (NHALF > 1) {
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                const float4 o = part[e][q];
                acc[q].x += o.x;
                acc[q].y += o.y;
                acc[q].z += o.z;
                acc[q].w += o.w;
            }
        }
        const size_t row = (size_t)s * p.H + (size_t)g * p.HG + h;
        const float gt0 = p.gates[row * 3], gt1 = p.gates[row * 3 + 1], gt2 = p.gates[row * 3 + 2];
        float4 r;
        r.x = gt0 * acc[0].x + gt1 * acc[1].x + gt2 * acc[2].x;
        r.y = gt0 * acc[0].y + gt1 * acc[1].y + gt2 * acc[2].y;
        r.z = gt0 * acc[0].z + gt1 * acc[1].z + gt2 * acc[2].z;
        r.w = gt0 * acc[0].w + gt1 * acc[1].w + gt2 * acc[2].w;
        *reinterpret_cast<float4*>(p.out + row * DV + c4) = r;
        if (c4 == 0 && p.lse) {
#pragma unroll
            for (int br = 0; br < 2; ++br) {
                const float lb = lsb[br][hl];
                p.lse[row * 3 + 1 + br] = lb == -INFINITY ? -INFINITY : lb * kLn2;
            }
            const float lc = p.lsecmp[sg * 16 + h];
            p.lse[row * 3] = lc == -INFINITY ? -INFINITY : lc * kLn2;
        }
    }
}

// workspace bytes for S sequences of at most Lmax tokens
inline size_t decode_ws_bytes(int64_t S, int64_t Lmax, int64_t G, int64_t l, int64_t d, int64_t lp,
                              int64_t w, int64_t n, int64_t DV) {
    const int64_t Cmax = Lmax >= l ? (Lmax - l) / d + 1 : 1;
    const int64_t NCH = (Cmax + 31) / 32;
    const int64_t NUV = n + (w + lp - 1) / lp + 1;
    auto a = [](size_t x) { return (x + 255) & ~size_t(255); };
    size_t o = 0;
    o += a((size_t)S * G * NCH * 16 * 4);
    o += a((size_t)S * G * NCH * kDecNBS * 16 * 4);
    o += a((size_t)(kDecMaxGrid * kDecW + S * G) * 16 * (DV + 4) * 4);
    o += a((size_t)S * G * 16 * 4);
    o += a((size_t)(kDecMaxGrid * kDecW + S * G) * 2 * 16 * (DV + 4) * 4);
    o += a((size_t)(S + 1) * 4);
    o += a((size_t)S * G * NUV * 4);
    return o;
}

}  // namespace nsa
