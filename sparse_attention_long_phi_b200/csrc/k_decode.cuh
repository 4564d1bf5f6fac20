// k_decode.cuh -- batched decode step (page "硬件对齐+原生训练！DeepSeek NSA打造高效
// 稀疏Attention", 效率分析 解码速度: per step NSA reads the compressed tokens, the
// selected blocks and the window, not the whole cache).
//
// One query per sequence at t = L-1 over packed varlen caches.  The step is
// HBM-bound: every cache row is read once.  The 16 heads of a GQA group are
// the M = 16 side of warp-level bf16 tensor-core products (mma.sync
// m16n8k16, fp32 accumulate).  The streaming kernels are persistent (one CTA
// per SM: 8 warps, 4 for the window stream).  Each warp pipelines K and V separately (the next
// chunk's K is in flight while this chunk's softmax and P.V run, its V while
// the next logits run) and keeps an online softmax.  Compressed stream: the
// chunks of 32 cache rows of all (seq, group) pairs form one sequence cut into
// equal contiguous ranges, one per warp; a warp streams its range across pair
// boundaries and writes a record per pair it touched at slot (warp index +
// seq*G + group), unique because consecutive pairs share at most one warp.
// The window stream takes the same per-warp ranges over the chunks that meet
// each pair's window, the selected stream over the pairs' selected blocks.
//   1. dec_cmp_stream   compressed cache: per segment (max, sum, unnormalised
//                       O); per chunk the head max and the per-head selection-
//                       block sums of exp(logit - chunk max), mapped with the
//                       overlap weights, so the importance scores can be
//                       normalised exactly once the row LSE is known.
//   2. dec_cmp_combine  per (seq, group): LSE, group importance scores (sum over
//                       heads and chunks of the block sums rescaled by
//                       exp(chunk max - LSE)), top-n by the CTA.
//   2b. dec_win_stream  the window's 32-token chunks, beside the combine (it does
//                       not need the selection; it waits for the combine before
//                       it exits).
//   3. dec_slcwin_stream  the selected blocks' chunks: logits, online softmax,
//                       P.V per warp.
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
constexpr int kDecMaxRecs = 64;      // records of a pair in the selected or the window stream
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
    float* part2;    // [grid3*8 + S*G][16][DV+4] per warp and pair of the selected stream
    float* partw;    // [gridw*4 + S*G][16][DV+4] per warp and pair of the window stream
    int* cpre;       // [S+1] compressed chunks (x G) before sequence s
    int* wpre;       // [S+1] window chunks (x G) before sequence s
    int Lmax, Cmax, NCH, NSmax;
    int grid1, grid3, gridw;
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

// -------------------------------------------------------------- step 2
// Every load that does not need the row LSE (chunk maxima, this thread's block
// sums) is issued before the first barrier; the records give the LSE in one
// batch of loads (their O is merged by the final step); the top-n runs on all
// warps and writes the row's selected block indices.
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
}

// -------------------------------------------------------------- step 2b
// The sliding window over the last w tokens of every (seq, group).  It does not
// depend on the selection, so it runs beside the combine: launched after it,
// small enough (four warps, one branch, at most 168 registers) to share an SM with a
// combine CTA, and waiting for the combine only before it exits, so that the
// kernels after it see the selection.  Items: the 32-token chunks meeting the
// window, of all (seq, group) pairs in one sequence cut into equal contiguous
// ranges, one per warp; per chunk the logits once, the window mask, an online
// softmax and P.V; a record per (warp, pair) at slot (warp index + seq*G + group).
// Shared memory: per warp two K/V stages (two chunks in flight) and a Q tile.
constexpr int kDecWinW = 4;          // warps per window-stream CTA

// 32-token chunks of a length-L sequence that meet its window [L-w, L-1]
__device__ __forceinline__ int dec_win_chunks(const DecParams& p, int L) {
    return (L - 1) / 32 - max(0, L - p.w) / 32 + 1;
}

template <int DK, int DV>
__host__ __device__ constexpr int dec_win_smem() {          // per warp: two K/V stages and a Q tile
    return kDecWinW * (2 * dec_stage_bytes<DK, DV>() + 16 * (DK * 2 + 16));
}

template <int DK, int DV>
__global__ void __launch_bounds__(128, 3) dec_win_stream(const DecParams p) {
    constexpr int KP = DK * 2 + 16, STG = dec_stage_bytes<DK, DV>(), REC = DV + 4;
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ int pre[kDecMaxSeqs + 1];
    __shared__ uint64_t kbar[kDecWinW][2], vbar[kDecWinW][2];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gr = lane >> 2, tg = lane & 3;
    uint8_t* stg0 = dsm + warp * 2 * STG;                 // stage b: K rows at stg0 + b*STG, V after them
    uint8_t* qs = dsm + kDecWinW * 2 * STG + warp * 16 * KP;   // this warp's [16][DK] Q tile
    if (threadIdx.x < kDecWinW * 2) {
        mbar_init(&kbar[threadIdx.x >> 1][threadIdx.x & 1], 1);
        mbar_init(&vbar[threadIdx.x >> 1][threadIdx.x & 1], 1);
    }
    fence_mbar_init();
    if (warp == 0) {
        int run = 0;
        for (int b0 = 0; b0 < p.S; b0 += 32) {
            const int s = b0 + lane;
            int cnt = 0, L, C;
            if (s < p.S && dec_seq_ok(p, s, L, C)) cnt = p.G * dec_win_chunks(p, L);
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
        for (int s = threadIdx.x; s <= p.S; s += blockDim.x) p.wpre[s] = pre[s];
    const long long N = pre[p.S];
    const int gw = blockIdx.x * kDecWinW + warp, W = gridDim.x * kDecWinW;
    long long x = dec_range_start(gw, N, W);
    const long long x1 = dec_range_start(gw + 1, N, W);
    const float cl = p.scale_log2;
    uint32_t kph = 0, vph = 0;                             // bit b: phase of stage b
    const uint64_t pol = l2_evict_first();
    const size_t kst = (size_t)p.G * DK, vst = (size_t)p.G * DV;
    struct Seg {
        int s, g, L, c, nw, u0;                      // chunk c of the pair's nw; its first token u0
        int64_t kvb;
    };
    auto locate = [&](long long xx, Seg& q) {
        int lo = 0, hi = p.S;                        // largest lo with pre[lo] <= xx
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (pre[mid] <= xx) lo = mid;
            else hi = mid;
        }
        int L, C;
        dec_seq_ok(p, lo, L, C);                     // lo holds chunks: its lengths passed
        const int nw = dec_win_chunks(p, L);
        const int r = (int)(xx - pre[lo]);
        q.s = lo;
        q.g = r / nw;
        q.L = L;
        q.c = r - q.g * nw;
        q.nw = nw;
        q.u0 = (max(0, L - p.w) / 32 + q.c) * 32;
        q.kvb = p.kv_off[lo];
    };
    // the item after q (x of q given): the pair's next chunk, or the next pair's first
    auto advance = [&](const Seg& q, long long xq, Seg& nx) {
        if (q.c + 1 < q.nw) {
            nx = q;
            ++nx.c;
            nx.u0 += 32;
        } else {
            locate(xq + 1, nx);
        }
    };
    auto issue = [&](const Seg& q, int b) {
        uint8_t* ks = stg0 + b * STG;
        warp_bulk_rows<DK>(ks, p.kcache + ((size_t)(q.kvb + q.u0) * p.G + q.g) * DK, kst, q.L - q.u0, &kbar[warp][b], pol);
        warp_bulk_rows<DV>(ks + 32 * KP, p.vcache + ((size_t)(q.kvb + q.u0) * p.G + q.g) * DV, vst, q.L - q.u0,
                           &vbar[warp][b], pol);
    };
    // Q of the group as a [16][DK] tile (rows >= HG zero), read with ldmatrix
    auto load_q_tile = [&](const Seg& q) {
        for (int e = lane; e < 16 * (DK / 8); e += 32) {
            const int h = e / (DK / 8), c8 = e % (DK / 8);
            int4 v = make_int4(0, 0, 0, 0);
            if (h < p.HG) v = *reinterpret_cast<const int4*>(p.q + ((size_t)q.s * p.H + (size_t)q.g * p.HG + h) * DK + c8 * 8);
            *reinterpret_cast<int4*>(qs + h * KP + c8 * 16) = v;
        }
        __syncwarp();
    };
    if (x < x1) {
        // two chunks in flight: chunk i in stage i & 1
        Seg cur, nx1;
        locate(x, cur);
        issue(cur, 0);
        if (x + 1 < x1) {
            advance(cur, x, nx1);
            issue(nx1, 1);
        }
        load_q_tile(cur);
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        float o[DV / 8][4];
#pragma unroll
        for (int nt = 0; nt < DV / 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
        for (int i = 0;; ++i) {
            const int b = i & 1;
            uint8_t* ks = stg0 + b * STG;
            if (!mbar_wait(&kbar[warp][b], (kph >> b) & 1, 0x405)) break;   // K of chunk i
            kph ^= 1u << b;
            __syncwarp();
            float sf[4][4];
            warp_logits_sa<DK>(smem_u32(qs), smem_u32(ks), sf);
            // keys u0 + k inside [L - w, L - 1]
            const int klo = cur.L - p.w - cur.u0, khi = cur.L - cur.u0;
            float mc0 = -INFINITY, mc1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = nt * 8 + tg * 2 + (e & 1);
                    const float v = (key >= klo && key < khi) ? sf[nt][e] * cl : -INFINITY;
                    sf[nt][e] = v;
                    if (e < 2) mc0 = fmaxf(mc0, v);
                    else mc1 = fmaxf(mc1, v);
                }
#pragma unroll
            for (int q2 = 1; q2 <= 2; q2 <<= 1) {
                mc0 = fmaxf(mc0, __shfl_xor_sync(0xffffffffu, mc0, q2));
                mc1 = fmaxf(mc1, __shfl_xor_sync(0xffffffffu, mc1, q2));
            }
            const float mn0 = fmaxf(m0, mc0), mn1 = fmaxf(m1, mc1);
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float v = sf[nt][e];
                    const float pv = v == -INFINITY ? 0.f : exp2f(v - (e < 2 ? mn0 : mn1));
                    sf[nt][e] = pv;
                    if (e < 2) s0 += pv;
                    else s1 += pv;
                }
#pragma unroll
            for (int q2 = 1; q2 <= 2; q2 <<= 1) {
                s0 += __shfl_xor_sync(0xffffffffu, s0, q2);
                s1 += __shfl_xor_sync(0xffffffffu, s1, q2);
            }
            const float a0 = mn0 == -INFINITY ? 1.f : exp2f(m0 - mn0);
            const float a1 = mn1 == -INFINITY ? 1.f : exp2f(m1 - mn1);
            m0 = mn0;
            m1 = mn1;
            l0 = l0 * a0 + s0;
            l1 = l1 * a1 + s1;
#pragma unroll
            for (int nt = 0; nt < DV / 8; ++nt) {
                o[nt][0] *= a0;
                o[nt][1] *= a0;
                o[nt][2] *= a1;
                o[nt][3] *= a1;
            }
            if (!mbar_wait(&vbar[warp][b], (vph >> b) & 1, 0x406)) break;   // V of chunk i
            vph ^= 1u << b;
            __syncwarp();
            warp_pv<DV>(sf, smem_u32(ks + 32 * KP), o);
            __syncwarp();
            const long long xi = x + i;
            const bool more = xi + 1 < x1;
            // stage b is free: chunk i + 2 goes there
            Seg nx2;
            if (xi + 2 < x1) {
                advance(nx1, xi + 1, nx2);
                issue(nx2, b);
            }
            if (!more || !(cur.s == nx1.s && cur.g == nx1.g)) {
                // this warp's record of (seq, group): (max, sum, -, -, O relative to max)
                const size_t sg = (size_t)cur.s * p.G + cur.g;
                float* rec = p.partw + ((size_t)gw + sg) * 16 * REC;
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
                if (more) load_q_tile(nx1);
            }
            if (!more) break;
            cur = nx1;
            nx1 = nx2;
        }
    }
    dep_wait();                                       // the combine: the kernels after this one read its selection
}

// -------------------------------------------------------------- step 3
template <int DK, int DV>
__host__ __device__ constexpr int dec_slcwin_smem() {        // staging + one Q tile per warp
    return kDecW * dec_stage_bytes<DK, DV>() + kDecW * 16 * (DK * 2 + 16);
}

// The selected branch.  Each warp owns a contiguous, equal range of the block
// slots (n per pair: the selection row, ascending, -1 padded); per pair it loads
// its own copy of Q and streams the chunks of the pair's blocks in its range,
// then writes one record at slot (warp index + seq*G + group), unique because
// consecutive pairs share at most one warp.
template <int DK, int DV>
__global__ void __launch_bounds__(256, 1) dec_slcwin_stream(const DecParams p) {
    constexpr int KP = DK * 2 + 16, STG = dec_stage_bytes<DK, DV>();
    extern __shared__ __align__(16) uint8_t dsm[];
    __shared__ uint64_t kbar[kDecW], vbar[kDecW];
    __shared__ int ulw[kDecW][33];                    // per warp: a batch's selected blocks, their count
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
    dep_wait();                                       // the combine's selections (through the window stream)
    uint32_t kph = 0, vph = 0;
    const uint64_t pol = l2_evict_first();
    const long long U = (long long)p.S * p.G * p.n;
    const int gw = blockIdx.x * kDecW + warp, W = gridDim.x * kDecW;
    long long x = dec_range_start(gw, U, W);
    const long long x1 = dec_range_start(gw + 1, U, W);
    const float cl = p.scale_log2;
    constexpr int REC = DV + 4;
    while (x < x1) {
        const size_t sg = (size_t)(x / p.n);
        const int ua = (int)(x % p.n);
        const int nslot = (int)min((long long)(p.n - ua), x1 - x);
        const int s = (int)(sg / p.G), g = (int)(sg % p.G);
        int L, C;
        const bool ok = dec_seq_ok(p, s, L, C);
        const int64_t kvb = ok ? p.kv_off[s] : 0;
        const size_t kst = (size_t)p.G * DK, vst = (size_t)p.G * DV;

        auto tok0 = [&](int blk, int i) { return blk * p.lp + (i & 1) * 32; };
        // rows past the cache are not read; the source stays inside the sequence
        auto issue_k = [&](int u0) {
            const int nv = min(32, L - u0);
            warp_bulk_rows<DK>(ks, p.kcache + ((size_t)(kvb + (nv > 0 ? u0 : 0)) * p.G + g) * DK, kst, nv, &kbar[warp], pol);
        };
        auto issue_v = [&](int u0) {
            const int nv = min(32, L - u0);
            warp_bulk_rows<DV>(vs, p.vcache + ((size_t)(kvb + (nv > 0 ? u0 : 0)) * p.G + g) * DV, vst, nv, &vbar[warp], pol);
        };
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        float o[DV / 8][4];
#pragma unroll
        for (int nt = 0; nt < DV / 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
        bool live = true, qready = false;
        // this range's blocks of the pair, 32 slots at a time (lane i: slot ua + b0 + i)
        for (int b0 = 0; b0 < nslot && live; b0 += 32) {
        {
            const int myu = (ok && b0 + lane < nslot) ? p.sel_idx[sg * p.n + ua + b0 + lane] : -1;
            const unsigned umask = __ballot_sync(0xffffffffu, myu >= 0);
            if (myu >= 0) ulw[warp][__popc(umask & ((1u << lane) - 1u))] = myu;
            if (lane == 0) ulw[warp][32] = __popc(umask);
        }
        __syncwarp();
        const int n = 2 * ulw[warp][32];                   // chunks of 32 tokens
        // block of chunk i: the (i/2)-th selected block of the batch
        auto block_of = [&](int i) { return ulw[warp][i >> 1]; };
        int bcur = n > 0 ? block_of(0) : 0;
        if (n > 0) {
            issue_k(tok0(bcur, 0));
            issue_v(tok0(bcur, 0));
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
            const int bnxt = more ? ((i & 1) ? block_of(i + 1) : bcur) : bcur;
            const int u0 = tok0(bcur, i);
            const int nval = min(32, L - u0);
            if (!mbar_wait(&kbar[warp], kph, 0x403)) {   // K of chunk i
                live = false;
                break;
            }
            kph ^= 1;
            __syncwarp();
            float sf[4][4];
            if (nval > 0) warp_logits_sa<DK>(smem_u32(qs), smem_u32(ks), sf);
            __syncwarp();
            if (more) issue_k(tok0(bnxt, i + 1));
            if (!mbar_wait(&vbar[warp], vph, 0x404)) {   // V of chunk i
                live = false;
                break;
            }
            vph ^= 1;
            __syncwarp();
            if (nval > 0) {
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
                const float mn0 = fmaxf(m0, mc0), mn1 = fmaxf(m1, mc1);
                float s0 = 0.f, s1 = 0.f;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float v = sf[nt][e];
                        const float pv = v == -INFINITY ? 0.f : exp2f(v - (e < 2 ? mn0 : mn1));
                        sf[nt][e] = pv;
                        if (e < 2) s0 += pv;
                        else s1 += pv;
                    }
#pragma unroll
                for (int q2 = 1; q2 <= 2; q2 <<= 1) {
                    s0 += __shfl_xor_sync(0xffffffffu, s0, q2);
                    s1 += __shfl_xor_sync(0xffffffffu, s1, q2);
                }
                const float a0 = mn0 == -INFINITY ? 1.f : exp2f(m0 - mn0);
                const float a1 = mn1 == -INFINITY ? 1.f : exp2f(m1 - mn1);
                m0 = mn0;
                m1 = mn1;
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
            }
            __syncwarp();
            if (more) issue_v(tok0(bnxt, i + 1));
            bcur = bnxt;
        }
        }
        if (!live) break;
        // this warp's record of the pair: (max, sum, -, -, O relative to max)
        float* rec = p.part2 + ((size_t)gw + sg) * 16 * REC;
        const int gr = lane >> 2;
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
        __syncwarp();                                  // the Q tile is reloaded for the next pair
        x += nslot;
    }
}

// -------------------------------------------------------------- step 4
// Per (seq, group) and eight heads (grid z): the records of all three
// branches merged in two phases of loads, each phase issued at once.  Phase 1:
// warp w takes the compressed records of head w (weight exp2(m - LSE) under
// the combine's LSE) and the selected/window records of two (branch, head)
// groups, 16 lanes per group (the branch max M, sum L and the weight
// exp2(m - M) / L of every record).  Phase 2: one thread per output float4
// (two for d_v = 64, each taking every other record) sums the weighted O of
// the records, eight of each kind per batch of loads; then
// out = sum_c g_c o_c and the LSEs.  256 CTAs of at most 128 registers per
// thread fit the GPU in one wave.
constexpr int kDecFinalHeads = 8;      // heads per dec_final CTA

template <int DV>
__global__ void __launch_bounds__(256, 2) dec_final(const DecParams p) {
    constexpr int REC = DV + 4, HQ = kDecFinalHeads, NOUT = HQ * DV / 4, NHALF = 256 / NOUT;
    static_assert(NHALF >= 1 && NHALF <= 2 && NHALF * NOUT == 256, "threads per output float4");
    __shared__ int recb[2][kDecMaxRecs];            // selected / window stream records
    __shared__ int recc[kDecMaxChunks];
    __shared__ int nrec[2], nrecc;
    __shared__ float wgt[kDecMaxRecs][2][HQ];       // selected/window record weight per branch and head
    __shared__ float wgc[kDecMaxChunks][HQ];        // compressed record weight per head
    __shared__ float lsb[2][HQ];                    // branch LSE (log2 units)
    __shared__ float4 part[NHALF > 1 ? NOUT : 1][3];   // the second thread's sums per output
    const int g = blockIdx.x, s = blockIdx.y, h0 = blockIdx.z * HQ;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int L, C;
    if (h0 >= p.HG || !dec_seq_ok(p, s, L, C)) return;
    const size_t sg = (size_t)s * p.G + g;
    const int nch = (C + 31) / 32;
    dep_wait();                                       // the selected branch's records
    if (warp == 0) {
        const long long X0 = (long long)sg * p.n;
        const int cnt = dec_record_list_warp(X0, X0 + p.n, (long long)p.S * p.G * p.n, p.grid3 * kDecW, recb[0],
                                             kDecMaxRecs);
        if (lane == 0) nrec[0] = cnt;
    } else if (warp == 2) {
        const int nw = dec_win_chunks(p, L);
        const long long X0 = (long long)p.wpre[s] + (long long)g * nw;
        const int cnt = dec_record_list_warp(X0, X0 + nw, (long long)p.wpre[p.S], p.gridw * kDecWinW, recb[1],
                                             kDecMaxRecs);
        if (lane == 0) nrec[1] = cnt;
    } else if (warp == 1) {
        int cnt = 0;
        if (nch > 0) {
            const long long X0 = (long long)p.cpre[s] + (long long)g * nch;
            cnt = dec_record_list_warp(X0, X0 + nch, p.cpre[p.S], p.grid1 * kDecW, recc, kDecMaxChunks);
        }
        if (lane == 0) nrecc = cnt;
    }
    __syncthreads();
    const int nrs = nrec[0], nrw = nrec[1], nrc = nrecc;
    {
        // compressed records of head h0 + warp (lane: records lane, lane + 32, ...) and
        // selected/window records of group (branch, head) gi (16 lanes), loads first
        const int hc = h0 + warp;
        const float lc = hc < p.HG ? p.lsecmp[sg * 16 + hc] : -INFINITY;
        const int gi = warp * 2 + (lane >> 4), sub = lane & 15;
        const int br = gi / HQ, hl = gi % HQ, h = h0 + hl;
        constexpr int PC = kDecMaxChunks / 32, PR = kDecMaxRecs / 16;
        float cm[PC], rm[PR], rl[PR];
#pragma unroll
        for (int k = 0; k < PC; ++k) {
            const int i = lane + 32 * k;
            cm[k] = (i < nrc && lc != -INFINITY) ? p.part1[((size_t)(recc[i] + sg) * 16 + hc) * REC] : -INFINITY;
        }
#pragma unroll
        for (int k = 0; k < PR; ++k) {
            const int i = sub + 16 * k;
            const bool use = i < (br ? nrw : nrs) && h < p.HG;
            const float* r = (br ? p.partw : p.part2) + (((size_t)recb[br][use ? i : 0] + sg) * 16 + (use ? h : 0)) * REC;
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
            if (i < (br ? nrw : nrs)) wgt[i][br][hl] = rm[k] == -INFINITY ? 0.f : exp2f(rm[k] - M) * inv;
        }
        if (sub == 0) lsb[br][hl] = Ls > 0.f ? M + log2f(Ls) : -INFINITY;
    }
    __syncthreads();
    // phase 2: output e (head h0 + e / (DV/4), channels c4 .. c4+3)
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
    const int nmax = max(max(nrs, nrw), nrc);
    for (int i0 = half; active && i0 < nmax; i0 += 8 * NHALF) {
        float4 vc[8], vs[8], vw[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int i = i0 + NHALF * k;
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            vc[k] = (i < nrc && wgc[i][hl] != 0.f)
                        ? *reinterpret_cast<const float4*>(p.part1 + ((size_t)(recc[i] + sg) * 16 + h) * REC + 4 + c4)
                        : z;
            vs[k] = (i < nrs && wgt[i][0][hl] != 0.f)
                        ? *reinterpret_cast<const float4*>(p.part2 + (((size_t)recb[0][i] + sg) * 16 + h) * REC + 4 + c4)
                        : z;
            vw[k] = (i < nrw && wgt[i][1][hl] != 0.f)
                        ? *reinterpret_cast<const float4*>(p.partw + (((size_t)recb[1][i] + sg) * 16 + h) * REC + 4 + c4)
                        : z;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int i = i0 + NHALF * k;
            fma4(acc[0], vc[k], i < nrc ? wgc[i][hl] : 0.f);
            fma4(acc[1], vs[k], i < nrs ? wgt[i][0][hl] : 0.f);
            fma4(acc[2], vw[k], i < nrw ? wgt[i][1][hl] : 0.f);
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
    (void)lp;
    (void)w;
    (void)n;
    auto a = [](size_t x) { return (x + 255) & ~size_t(255); };
    size_t o = 0;
    o += a((size_t)S * G * NCH * 16 * 4);
    o += a((size_t)S * G * NCH * kDecNBS * 16 * 4);
    o += a((size_t)(kDecMaxGrid * kDecW + S * G) * 16 * (DV + 4) * 4);
    o += a((size_t)S * G * 16 * 4);
    o += a((size_t)(kDecMaxGrid * kDecW + S * G) * 16 * (DV + 4) * 4);
    o += a((size_t)(kDecMaxGrid * kDecWinW + S * G) * 16 * (DV + 4) * 4);
    o += a((size_t)(S + 1) * 4);
    o += a((size_t)(S + 1) * 4);
    return o;
}

}  // namespace nsa
