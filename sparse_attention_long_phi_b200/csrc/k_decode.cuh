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
    float* ocmp;     // [S*G][16][DV]             normalised compressed-branch output
    float* lsecmp;   // [S*G][16]                 log2 units
    float* part2;    // [grid3 + S*G][2][16][DV+4] per segment and branch (selected, window)
    int* cpre;       // [S+1] compressed chunks (x G) before sequence s
    int Lmax, Cmax, NCH, NUV, NSmax;
    int grid1, grid3;
};

template <int DK, int DV>
__host__ __device__ constexpr int dec_stage_bytes() {      // one warp: 32 K rows + 32 V rows
    return 32 * ((DK * 2 + 16) + (DV * 2 + 16));
}
template <int DK, int DV>
__host__ __device__ constexpr int dec_stream_smem() {      // staging (merge area aliased) + P tiles
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
// record slots of items [X0, X1) (X1 > X0): CTAs with a non-empty range
// among those holding them; returns the count, slots b + sg into out[]
__device__ __forceinline__ int dec_record_ctas(long long X0, long long X1, long long N, int grid, int* out, int cap) {
    const int bf = dec_cta_of(X0, N, grid), bl = dec_cta_of(X1 - 1, N, grid);
    int cnt = 0;
    for (int b = bf; b <= bl && cnt < cap; ++b)
        if (dec_range_start(b + 1, N, grid) > dec_range_start(b, N, grid)) out[cnt++] = b;
    return cnt;
}

// Merge the 8 warps' online-softmax states (rows gr, gr+8 per lane) into one
// record [16][DV+4] = (max, sum, -, -, O relative to max).  `mrg` is a
// [8][16][DV] fp32 scratch; wm/wl [8][16].  Ends with a barrier.
template <int DV>
__device__ __forceinline__ void dec_merge_record(float m0, float m1, float l0, float l1, const float (&o)[DV / 8][4],
                                                 float* mrg, float (*wm)[16], float (*wl)[16], float* rec) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gr = lane >> 2, tg = lane & 3;
    if (tg == 0) {
        wm[warp][gr] = m0;
        wm[warp][gr + 8] = m1;
        wl[warp][gr] = l0;
        wl[warp][gr + 8] = l1;
    }
    __syncthreads();
    {
        float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
        for (int w2 = 0; w2 < kDecW; ++w2) {
            M0 = fmaxf(M0, wm[w2][gr]);
            M1 = fmaxf(M1, wm[w2][gr + 8]);
        }
        const float f0 = m0 == -INFINITY ? 0.f : exp2f(m0 - M0);
        const float f1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M1);
#pragma unroll
        for (int nt = 0; nt < DV / 8; ++nt) {
            const int cc = nt * 8 + tg * 2;
            *reinterpret_cast<float2*>(mrg + (warp * 16 + gr) * DV + cc) = make_float2(o[nt][0] * f0, o[nt][1] * f0);
            *reinterpret_cast<float2*>(mrg + (warp * 16 + gr + 8) * DV + cc) = make_float2(o[nt][2] * f1, o[nt][3] * f1);
        }
    }
    __syncthreads();
    constexpr int REC = DV + 4;
    for (int e = threadIdx.x; e < 16 * (DV / 4); e += blockDim.x) {
        const int h = e / (DV / 4), c4 = (e % (DV / 4)) * 4;
        float4 a = *reinterpret_cast<const float4*>(mrg + h * DV + c4);
#pragma unroll
        for (int w2 = 1; w2 < kDecW; ++w2) {       // fixed order: deterministic
            const float4 b = *reinterpret_cast<const float4*>(mrg + (w2 * 16 + h) * DV + c4);
            a.x += b.x;
            a.y += b.y;
            a.z += b.z;
            a.w += b.w;
        }
        *reinterpret_cast<float4*>(rec + h * REC + 4 + c4) = a;
    }
    if (threadIdx.x < 16) {
        const int h = threadIdx.x;
        float M = -INFINITY;
        for (int w2 = 0; w2 < kDecW; ++w2) M = fmaxf(M, wm[w2][h]);
        float Ls = 0.f;
        for (int w2 = 0; w2 < kDecW; ++w2)
            if (wm[w2][h] != -INFINITY) Ls += wl[w2][h] * exp2f(wm[w2][h] - M);
        rec[h * REC] = M;
        rec[h * REC + 1] = Ls;
    }
    __syncthreads();
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
// Every load that does not need the row LSE (records, chunk maxima, this
// thread's block sums) is issued before the first barrier, so the kernel
// waits about one memory round trip; the top-n runs on all 8 warps.
template <int DV>
__global__ void __launch_bounds__(256) dec_cmp_combine(const DecParams p) {
    constexpr int REC = DV + 4;
    extern __shared__ float csm[];                     // ifac [256][16], fac [NCH][16], pg [NSmax]
    __shared__ float lse2[16];
    __shared__ int recb[kDecMaxChunks];
    __shared__ int nrec;
    __shared__ int tsm[256 + 16 + 8 * 8 + 32];       // top-n scratch
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
    if (threadIdx.x == 0) {
        int cnt = 0;
        if (nch > 0) {
            const long long X0 = (long long)p.cpre[s] + (long long)g * nch;
            cnt = dec_record_ctas(X0, X0 + nch, p.cpre[p.S], p.grid1 * kDecW, recb, kDecMaxChunks);
        }
        nrec = cnt;
    }
    float* ifac = csm;
    float* fac = csm + kDecMaxChunks * 16;
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
        const int h = threadIdx.x >> 4, sub = threadIdx.x & 15;
        float M = -INFINITY, Ls = 0.f;
        for (int i0 = sub; i0 < nr; i0 += 64) {
            float rm[4], rl[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = i0 + 16 * k;
                const float* r = p.part1 + ((size_t)(recb[i < nr ? i : 0] + sg) * 16 + h) * REC;
                rm[k] = i < nr ? r[0] : -INFINITY;
                rl[k] = i < nr ? r[1] : 0.f;
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
        if (sub == 0) {
            lse2[h] = l2;
            p.lsecmp[sg * 16 + h] = l2;
        }
        for (int i = sub; i < nr; i += 16) {
            const float m = p.part1[((size_t)(recb[i] + sg) * 16 + h) * REC];
            ifac[i * 16 + h] = (m != -INFINITY && l2 != -INFINITY) ? exp2f(m - l2) : 0.f;
        }
    }
    __syncthreads();
    // per chunk and head: exp2(chunk max - LSE); heads past HG do not score
    for (int e = threadIdx.x; e < nch * 16; e += blockDim.x) {
        const int h = e & 15;
        fac[e] = (h < p.HG && lse2[h] != -INFINITY) ? exp2f(fac[e] - lse2[h]) : 0.f;
    }
    // o_cmp = sum over records of O exp2(m - LSE)
    for (int e = threadIdx.x; e < 16 * (DV / 4); e += blockDim.x) {
        const int h = e / (DV / 4), c4 = (e % (DV / 4)) * 4;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i0 = 0; i0 < nr; i0 += 8) {
            float4 v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                v[k] = i0 + k < nr ? *reinterpret_cast<const float4*>(p.part1 + ((size_t)(recb[i0 + k] + sg) * 16 + h) * REC + 4 + c4)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float f = i0 + k < nr ? ifac[(i0 + k) * 16 + h] : 0.f;
                a.x += v[k].x * f;
                a.y += v[k].y * f;
                a.z += v[k].z * f;
                a.w += v[k].w * f;
            }
        }
        *reinterpret_cast<float4*>(p.ocmp + (sg * 16 + h) * DV + c4) = a;
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
    topn_row_cta_radix<256>(pg, t, p.n, p.lp, p.fi, p.fl, p.sel_idx + sg * p.n, tsm);
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

// -------------------------------------------------------------- step 3
template <int DK, int DV>
__global__ void __launch_bounds__(256, 1) dec_slcwin_stream(const DecParams p) {
    constexpr int KP = DK * 2 + 16, STG = dec_stage_bytes<DK, DV>();
    extern __shared__ __align__(16) uint8_t dsm[];
    float* mrg = reinterpret_cast<float*>(dsm);
    uint8_t* qs = dsm + kDecW * STG;                      // [16][DK] Q tile, pitch DK*2+16
    static_assert(16 * (DK * 2 + 16) <= kDecW * 16 * 33 * 4, "Q tile");
    __shared__ float wm[kDecW][16], wl[kDecW][16];
    __shared__ int ulist[kDecMaxUnits], uflag[kDecMaxUnits];
    __shared__ int selbuf[32];
    __shared__ int nunits;
    __shared__ uint64_t kbar[kDecW], vbar[kDecW];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tg = lane & 3;
    uint8_t* ks = dsm + warp * STG;
    uint8_t* vs = ks + 32 * KP;
    if (threadIdx.x < kDecW) {
        mbar_init(&kbar[threadIdx.x], 1);
        mbar_init(&vbar[threadIdx.x], 1);
    }
    fence_mbar_init();
    __syncthreads();
    dep_launch();
    dep_wait();                                       // sel_idx and o_cmp of the combine
    uint32_t kph = 0, vph = 0;
    const uint64_t pol = l2_evict_first();
    const long long U = (long long)p.S * p.G * p.NUV;     // unit slots, NUV per (seq, group)
    const int b = blockIdx.x;
    long long x = dec_range_start(b, U, gridDim.x);
    const long long x1 = dec_range_start(b + 1, U, gridDim.x);
    const float cl = p.scale_log2;
    while (x < x1) {
        const size_t sg = (size_t)(x / p.NUV);
        const int ua = (int)(x % p.NUV);
        const int nslot = (int)min((long long)(p.NUV - ua), x1 - x);
        const int s = (int)(sg / p.G), g = (int)(sg % p.G);
        int L, C;
        const bool ok = dec_seq_ok(p, s, L, C);
        if (warp == 0) {                                  // unit list of (s, g)
            if (ok && lane < p.n) selbuf[lane] = p.sel_idx[sg * p.n + lane];
            __syncwarp();
            if (lane == 0) nunits = ok ? dec_units(p, selbuf, L, ulist, uflag) : 0;
        }
        // Q of the group as a [16][DK] tile (rows >= HG zero), read with ldmatrix
        for (int e = threadIdx.x; e < 16 * (DK / 8); e += blockDim.x) {
            const int h = e / (DK / 8), c8 = e % (DK / 8);
            int4 v = make_int4(0, 0, 0, 0);
            if (h < p.HG) v = *reinterpret_cast<const int4*>(p.q + ((size_t)s * p.H + (size_t)g * p.HG + h) * DK + c8 * 8);
            *reinterpret_cast<int4*>(qs + h * KP + c8 * 16) = v;
        }
        __syncthreads();
        const int n = 2 * max(0, min(ua + nslot, nunits) - ua);   // chunks of 32 tokens
        const int64_t kvb = ok ? p.kv_off[s] : 0;
        const size_t kst = (size_t)p.G * DK, vst = (size_t)p.G * DV;
        auto tok0 = [&](int i) { return ulist[ua + (i >> 1)] * p.lp + (i & 1) * 32; };
        // rows past the cache are not read; the source stays inside the sequence
        auto issue_k = [&](int i) {
            const int u0 = tok0(i), nv = min(32, L - u0);
            warp_bulk_rows<DK>(ks, p.kcache + ((size_t)(kvb + (nv > 0 ? u0 : 0)) * p.G + g) * DK, kst, nv, &kbar[warp], pol);
        };
        auto issue_v = [&](int i) {
            const int u0 = tok0(i), nv = min(32, L - u0);
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
        int i = warp;
        if (i < n) {
            issue_k(i);
            issue_v(i);
        }
        for (; i < n; i += kDecW) {
            const bool more = i + kDecW < n;
            const int u0 = tok0(i);
            const bool insel = uflag[ua + (i >> 1)] != 0;
            const int nval = min(32, L - u0);
            // warp-uniform: does the chunk hold keys of each branch?
            const bool has_sel = insel && nval > 0;
            const bool has_win = nval > 0 && u0 + nval - 1 >= wlo;
            if (!mbar_wait(&kbar[warp], kph, 0x403)) break;   // K of chunk i
            kph ^= 1;
            __syncwarp();
            float sf[4][4];
            if (has_sel || has_win) warp_logits_sa<DK>(smem_u32(qs), smem_u32(ks), sf);
            __syncwarp();
            if (more) issue_k(i + kDecW);
            if (!mbar_wait(&vbar[warp], vph, 0x404)) break;   // V of chunk i
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
            if (more) issue_v(i + kDecW);
        }
        float* rec = p.part2 + ((size_t)b + sg) * 2 * 16 * (DV + 4);
        dec_merge_record<DV>(m[0][0], m[0][1], l[0][0], l[0][1], o[0], mrg, wm, wl, rec);
        dec_merge_record<DV>(m[1][0], m[1][1], l[1][0], l[1][1], o[1], mrg, wm, wl, rec + 16 * (DV + 4));
        x += nslot;
    }
}

// -------------------------------------------------------------- step 4
// One thread per output float4: it merges its head's records of both
// branches itself (one pass, running max), so the only barrier is the one
// that publishes the record list.
template <int DV>
__global__ void __launch_bounds__(256) dec_final(const DecParams p) {
    constexpr int REC = DV + 4;
    __shared__ int recb[kDecMaxUnits];
    __shared__ int nrec;
    const int g = blockIdx.x, s = blockIdx.y;
    int L, C;
    if (!dec_seq_ok(p, s, L, C)) return;
    const size_t sg = (size_t)s * p.G + g;
    dep_wait();                                       // the selected/window records
    if (threadIdx.x == 0) {
        const long long X0 = (long long)sg * p.NUV;
        nrec = dec_record_ctas(X0, X0 + p.NUV, (long long)p.S * p.G * p.NUV, p.grid3, recb, kDecMaxUnits);
    }
    __syncthreads();
    const int nr = nrec;
    for (int e = threadIdx.x; e < p.HG * (DV / 4); e += blockDim.x) {
        const int h = e / (DV / 4), c4 = (e % (DV / 4)) * 4;
        const size_t row = (size_t)s * p.H + g * p.HG + h;
        const float4 oc = *reinterpret_cast<const float4*>(p.ocmp + (sg * 16 + h) * DV + c4);
        const float gt0 = p.gates[row * 3], gt1 = p.gates[row * 3 + 1], gt2 = p.gates[row * 3 + 2];
        float M[2] = {-INFINITY, -INFINITY}, Ls[2] = {0.f, 0.f};
        float4 O[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
        for (int i0 = 0; i0 < nr; i0 += 4) {
            // every load of four records (both branches) in flight before the merge
            float rm[4][2], rl[4][2];
            float4 rv[4][2];
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
                for (int br = 0; br < 2; ++br) {
                    const bool in = i0 + k < nr;
                    const float* r = p.part2 + ((((size_t)recb[in ? i0 + k : 0] + sg) * 2 + br) * 16 + h) * REC;
                    rm[k][br] = in ? r[0] : -INFINITY;
                    rl[k][br] = in ? r[1] : 0.f;
                    rv[k][br] = in ? *reinterpret_cast<const float4*>(r + 4 + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
                for (int br = 0; br < 2; ++br) {
                    const float m = rm[k][br];
                    if (m == -INFINITY) continue;
                    const float4 v = rv[k][br];
                    const float Mn = fmaxf(M[br], m);
                    const float a = exp2f(M[br] - Mn), f = exp2f(m - Mn);   // M = -inf first: a = 0
                    Ls[br] = Ls[br] * a + rl[k][br] * f;
                    O[br].x = O[br].x * a + v.x * f;
                    O[br].y = O[br].y * a + v.y * f;
                    O[br].z = O[br].z * a + v.z * f;
                    O[br].w = O[br].w * a + v.w * f;
                    M[br] = Mn;
                }
        }
        float inv[2];
#pragma unroll
        for (int br = 0; br < 2; ++br) inv[br] = Ls[br] > 0.f ? 1.f / Ls[br] : 0.f;
        float4 r;
        r.x = gt0 * oc.x + gt1 * O[0].x * inv[0] + gt2 * O[1].x * inv[1];
        r.y = gt0 * oc.y + gt1 * O[0].y * inv[0] + gt2 * O[1].y * inv[1];
        r.z = gt0 * oc.z + gt1 * O[0].z * inv[0] + gt2 * O[1].z * inv[1];
        r.w = gt0 * oc.w + gt1 * O[0].w * inv[0] + gt2 * O[1].w * inv[1];
        *reinterpret_cast<float4*>(p.out + row * DV + c4) = r;
        if (c4 == 0 && p.lse) {
#pragma unroll
            for (int br = 0; br < 2; ++br)
                p.lse[row * 3 + 1 + br] = Ls[br] > 0.f ? (M[br] + log2f(Ls[br])) * kLn2 : -INFINITY;
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
    o += a((size_t)S * G * 16 * DV * 4);
    o += a((size_t)S * G * 16 * 4);
    o += a((size_t)(kDecMaxGrid + S * G) * 2 * 16 * (DV + 4) * 4);
    o += a((size_t)(S + 1) * 4);
    (void)NUV;
    return o;
}

}  // namespace nsa
