// k_topn.cuh -- top-n block selection (page "硬件对齐+原生训练！DeepSeek NSA打造高效
// 稀疏Attention", Top-n 块选择; hyperparameter paragraph: 1 initial + 2 local
// blocks always active).
//
// One warp per (batch, token, group).  Candidates are the selection blocks
// 0 .. b_t = floor(t/l').  With at most n candidates all are taken.
// Otherwise blocks 0..fi-1 and b_t-fl+1..b_t are kept and the remaining
// n - fi - fl are the highest importance scores among the other candidates,
// ties to the lower block index (decision taken on the fp32 scores).  The
// output row is ascending and padded with -1.
#pragma once
#include "nsa_dev.cuh"

namespace nsa {

constexpr int kTopnPerLane = 64;   // up to 2048 scored candidates per row

__device__ __forceinline__ int warp_sort_asc(int v, int lane) {
    // bitonic sort of one int per lane across the warp, ascending by lane
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            int o = __shfl_xor_sync(0xffffffffu, v, j);
            bool up = ((lane & k) == 0);
            bool lower = ((lane & j) == 0);
            int mn = min(v, o), mx = max(v, o);
            v = (lower == up) ? mn : mx;
        }
    }
    return v;
}

// bitonic sort of one value per lane across the warp, descending by lane
template <typename U>
__device__ __forceinline__ U warp_sort_desc(U v, int lane) {
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const U o = __shfl_xor_sync(0xffffffffu, v, j);
            const bool up = ((lane & k) == 0);
            const bool lower = ((lane & j) == 0);
            const U mn = v < o ? v : o, mx = v < o ? o : v;
            v = (lower == up) ? mx : mn;
        }
    }
    return v;
}

// Top-n of one row of importance scores `row` (global or shared memory) for
// query t, by one warp; writes n ascending indices (-1 padded) to `out`.
// PL candidates per lane: rows of at most 32*PL scored candidates.
//
// Candidate j sits in lane (j - lo) % 32, slot (j - lo) / 32.  Scores are
// mapped to keys that order like the scores (+0 and -0 equal; a negative
// score, the padding, or a NaN maps to 0 and is never taken).  Each lane keeps
// its two best untaken candidates (ties: lower slot = lower j first); a round
// takes the warp's largest head key (__reduce_max_sync) and, among the lanes
// holding it, the lowest j (__reduce_min_sync): the highest score, ties to the
// lower block index.  The winning lane pops its head and rescans its slots
// when both cached entries are used up.
//
// Most rows skip those rounds: with theta the R-th largest of the 32 lane
// maxima, at least R candidates have key >= theta, so every winner does.  When
// at most 32 candidates reach theta they are gathered into `wbuf` (32 slots of
// this warp) as (key, ~j) and one descending warp sort leaves the winners, in
// order, in lanes 0..R-1.  The rounds above are the fallback for rows with
// more (ties at theta) or with theta = 0.
__device__ __forceinline__ uint32_t topn_key(float x) {
    return x > 0.f ? __float_as_uint(x) + 1u : (x == 0.f ? 1u : 0u);
}

template <int PL = kTopnPerLane>
__device__ __forceinline__ void topn_row_warp(const float* row, int t, int n, int lp, int fi, int fl,
                                              int32_t* out, int lane, unsigned long long* wbuf) {
    static_assert(PL <= 64, "taken mask is 64 bits");
    const int bt = t / lp;
    const int ncand = bt + 1;
    if (ncand <= n) {
        if (lane < n) out[lane] = lane < ncand ? lane : -1;
        return;
    }
    const int lo = fi, hi = bt - fl;             // scored candidates lo..hi
    const int R = n - fi - fl;
    // every lane loads all its slots from in-bounds addresses (slots past hi
    // re-read row[hi]) so that the loads carry no predicate and are all in
    // flight together; the slots past hi are masked afterwards
    float raw[PL];
#pragma unroll
    for (int k = 0; k < PL; ++k) raw[k] = row[min(lo + lane + 32 * k, hi)];
    uint32_t key[PL];
    uint32_t lmax = 0;
#pragma unroll
    for (int k = 0; k < PL; ++k) {
        const int j = lo + lane + 32 * k;
        key[k] = (j <= hi) ? topn_key(raw[k]) : 0u;
        lmax = max(lmax, key[k]);
    }
    int mine = 0x7fffffff;
    bool done = R <= 0;                          // only forced blocks
    const uint32_t theta = done ? 0u : __shfl_sync(0xffffffffu, warp_sort_desc(lmax, lane), R - 1);
    if (theta > 0u) {
        int cnt = 0;
#pragma unroll
        for (int k = 0; k < PL; ++k) cnt += key[k] >= theta;
        const int total = (int)__reduce_add_sync(0xffffffffu, (unsigned)cnt);
        if (total <= 32) {
            int pos = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, pos, o);
                if (lane >= o) pos += y;
            }
            pos -= cnt;                            // exclusive prefix
#pragma unroll
            for (int k = 0; k < PL; ++k)
                if (key[k] >= theta)
                    wbuf[pos++] = ((unsigned long long)key[k] << 32) | (uint32_t)~(uint32_t)(lo + lane + 32 * k);
            __syncwarp();
            unsigned long long c = lane < total ? wbuf[lane] : 0ull;
            __syncwarp();                          // wbuf is free for the warp's next row
            c = warp_sort_desc(c, lane);
            if (lane < R) mine = (int)~(uint32_t)c;
            done = true;
        }
    }
    if (!done) {
        uint64_t taken = 0;
        uint32_t c0 = 0, c1 = 0;                     // cached keys, c0 >= c1
        int s0 = 0, s1 = 0;                          // their slots
        auto rescan = [&]() {
            c0 = c1 = 0;
#pragma unroll
            for (int k = 0; k < PL; ++k) {
                const uint32_t kk = ((taken >> k) & 1ull) ? 0u : key[k];
                const bool g0 = kk > c0, g1 = kk > c1;   // strict: the lower slot stays ahead
                c1 = g0 ? c0 : (g1 ? kk : c1);
                s1 = g0 ? s0 : (g1 ? k : s1);
                c0 = g0 ? kk : c0;
                s0 = g0 ? k : s0;
            }
        };
        rescan();
        for (int it = 0; it < R; ++it) {
            const uint32_t mx = __reduce_max_sync(0xffffffffu, c0);
            if (mx == 0u) break;                     // warp-uniform: nothing left to take
            const uint32_t mj = (c0 == mx) ? (uint32_t)(lo + lane + 32 * s0) : 0xffffffffu;
            const uint32_t bj = __reduce_min_sync(0xffffffffu, mj);
            if (mj == bj) {                          // this lane holds the winner
                taken |= 1ull << s0;
                c0 = c1;
                s0 = s1;
                c1 = 0;
                if (c0 == 0u) rescan();
            }
            if (lane == it) mine = (int)bj;
        }
    }
    // lanes R .. R+fi+fl-1 carry the forced blocks
    if (lane >= R && lane < R + fi) mine = lane - R;
    if (lane >= R + fi && lane < R + fi + fl) mine = bt - fl + 1 + (lane - R - fi);
    const int srt = warp_sort_asc(mine, lane);
    if (lane < n) out[lane] = (srt == 0x7fffffff) ? -1 : srt;
}

// The same selection by a whole CTA of NW warps, for long candidate rows in
// shared memory: warp w takes the top R of its contiguous slice of the scored
// candidates, warp 0 then takes the top R of the NW*R survivors (ordered by
// score, then lower index, exactly as above).  sv/si: NW*16 scratch slots.
// Called by every thread of the CTA.
template <int NW>
__device__ __forceinline__ void topn_row_cta(const float* row, int t, int n, int lp, int fi, int fl,
                                             int32_t* out, float* sv, int* si) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bt = t / lp;
    const int ncand = bt + 1;
    if (ncand <= n) {
        if (threadIdx.x < n) out[threadIdx.x] = (int)threadIdx.x < ncand ? (int)threadIdx.x : -1;
        return;
    }
    const int lo = fi, hi = bt - fl;
    const int R = n - fi - fl;
    const int M = hi - lo + 1;
    const int per = (M + NW - 1) / NW;
    constexpr int PL = (kTopnPerLane * 32 / NW + 31) / 32;      // values per lane per slice
    const int s0 = lo + warp * per, s1 = min(hi + 1, s0 + per);
    float v[PL];
#pragma unroll
    for (int k = 0; k < PL; ++k) {
        const int j = s0 + lane + 32 * k;
        v[k] = j < s1 ? row[j] : -1.f;              // scores are >= 0
    }
    for (int it = 0; it < R; ++it) {
        float bv = -2.f;
        int bk = 0;
#pragma unroll
        for (int k = 0; k < PL; ++k)
            if (v[k] > bv) {
                bv = v[k];
                bk = k;
            }
        int bj = s0 + lane + 32 * bk;
        if (bv < -0.5f) bj = 0x7fffffff;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
            if (ov > bv || (ov == bv && oj < bj)) {
                bv = ov;
                bj = oj;
            }
        }
        if (bj != 0x7fffffff && ((bj - s0) & 31) == lane) {
            const int kk = (bj - s0) >> 5;
#pragma unroll
            for (int k = 0; k < PL; ++k)
                if (k == kk) v[k] = -1.f;
        }
        if (lane == 0) {
            sv[warp * 16 + it] = bj == 0x7fffffff ? -2.f : bv;
            si[warp * 16 + it] = bj;
        }
    }
    __syncthreads();
    if (warp == 0) {
        constexpr int Q = (NW * 16 + 31) / 32;
        float w[Q];
        int wi[Q];
#pragma unroll
        for (int k = 0; k < Q; ++k) {
            const int e = lane + 32 * k, ww = e / 16, r = e % 16;
            const bool ok = ww < NW && r < R;
            w[k] = ok ? sv[e] : -2.f;
            wi[k] = ok ? si[e] : 0x7fffffff;
        }
        int mine = 0x7fffffff;
        for (int it = 0; it < R; ++it) {
            float bv = -2.f;
            int bj = 0x7fffffff, bk = -1;
#pragma unroll
            for (int k = 0; k < Q; ++k)
                if (w[k] > bv || (w[k] == bv && wi[k] < bj)) {
                    bv = w[k];
                    bj = wi[k];
                    bk = k;
                }
            if (bv < -0.5f) bj = 0x7fffffff;
            int owner = bk >= 0 ? lane : 32;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
                const int oo = __shfl_xor_sync(0xffffffffu, owner, o);
                if (ov > bv || (ov == bv && oj < bj)) {
                    bv = ov;
                    bj = oj;
                    owner = oo;
                }
            }
            if (bj != 0x7fffffff && owner == lane) {
#pragma unroll
                for (int k = 0; k < Q; ++k)
                    if (wi[k] == bj) w[k] = -2.f;
            }
            if (lane == it) mine = bj;
        }
        if (lane >= R && lane < R + fi) mine = lane - R;
        if (lane >= R + fi && lane < R + fi + fl) mine = bt - fl + 1 + (lane - R - fi);
        const int srt = warp_sort_asc(mine, lane);
        if (lane < n) out[lane] = (srt == 0x7fffffff) ? -1 : srt;
    }
}

// The same selection by a whole CTA of NT threads, for rows of up to 2048
// candidates.  For scores >= 0 the fp32 bit pattern orders like the value (-0
// counts as +0); a candidate's key is that pattern + 1, and 0 marks a score
// that is never selected (negative, NaN, or already taken).  Each warp takes
// the top R of its candidates (j = lo + thread + NT*k) one at a time: the
// warp-wide maximum key and, among the candidates holding it, the lowest block
// index are single reductions (redux.sync); warp 0 then takes the top R of the
// warps' lists the same way.  Ties therefore go to the lower block index, the
// rule of the iterative maximum above.
// sm: >= NT/32 * 32 * 2 + 2 ints of shared memory.
template <int NT>
__device__ __forceinline__ void topn_row_cta_redux(const float* row, int t, int n, int lp, int fi, int fl,
                                                   int32_t* out, int* sm) {
    constexpr int NW = NT / 32, PL = (32 * kTopnPerLane + NT - 1) / NT;
    unsigned* wkey = reinterpret_cast<unsigned*>(sm);   // [NW][32] each warp's picks (key)
    int* widx = sm + NW * 32;                           // [NW][32]                (block)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bt = t / lp;
    const int ncand = bt + 1;
    if (ncand <= n) {
        if (tid < n) out[tid] = tid < ncand ? tid : -1;
        return;
    }
    const int lo = fi, hi = bt - fl;
    const int R = n - fi - fl;
    unsigned key[PL];
#pragma unroll
    for (int k = 0; k < PL; ++k) {
        const int j = lo + tid + NT * k;
        const float v = j <= hi ? row[j] : -1.f;
        key[k] = v >= 0.f ? (__float_as_uint(v) & 0x7fffffffu) + 1u : 0u;   // 0 for negative or NaN
    }
    // the warp's top R, best first
    for (int it = 0; it < R; ++it) {
        unsigned lm = 0;
#pragma unroll
        for (int k = 0; k < PL; ++k) lm = max(lm, key[k]);
        const unsigned M = __reduce_max_sync(0xffffffffu, lm);
        unsigned jm = 0xffffffffu;
        if (M != 0u) {
#pragma unroll
            for (int k = PL - 1; k >= 0; --k)
                if (key[k] == M) jm = (unsigned)(lo + tid + NT * k);
        }
        const unsigned J = __reduce_min_sync(0xffffffffu, jm);
        if (M != 0u && jm == J) {
#pragma unroll
            for (int k = 0; k < PL; ++k)
                if ((unsigned)(lo + tid + NT * k) == J) key[k] = 0u;
        }
        if (lane == 0) {
            wkey[warp * 32 + it] = M;
            widx[warp * 32 + it] = M != 0u ? (int)J : 0x7fffffff;
        }
    }
    __syncthreads();
    if (warp == 0) {
        // the warps' lists: lane l holds entries l, l + 32, ... of the NW x R candidates
        constexpr int Q = (NW * 32 + 31) / 32;
        unsigned ck[Q];
        int ci[Q];
#pragma unroll
        for (int q = 0; q < Q; ++q) {
            const int e = lane + 32 * q, ww = e / 32, r = e % 32;
            const bool ok = ww < NW && r < R;
            ck[q] = ok ? wkey[e] : 0u;
            ci[q] = ok ? widx[e] : 0x7fffffff;
        }
        int mine = 0x7fffffff;
        for (int it = 0; it < R; ++it) {
            unsigned lm = 0;
#pragma unroll
            for (int q = 0; q < Q; ++q) lm = max(lm, ck[q]);
            const unsigned M = __reduce_max_sync(0xffffffffu, lm);
            unsigned jm = 0xffffffffu;
            if (M != 0u) {
#pragma unroll
                for (int q = 0; q < Q; ++q)
                    if (ck[q] == M) jm = min(jm, (unsigned)ci[q]);
            }
            const unsigned J = __reduce_min_sync(0xffffffffu, jm);
            if (M != 0u && jm == J) {
#pragma unroll
                for (int q = 0; q < Q; ++q)
                    if ((unsigned)ci[q] == J) ck[q] = 0u;
            }
            if (lane == it) mine = M != 0u ? (int)J : 0x7fffffff;
        }
        if (lane >= R && lane < R + fi) mine = lane - R;
        if (lane >= R + fi && lane < R + fi + fl) mine = bt - fl + 1 + (lane - R - fi);
        const int srt = warp_sort_asc(mine, lane);
        if (lane < n) out[lane] = (srt == 0x7fffffff) ? -1 : srt;
    }
}

// one CTA per (batch, token, group) item, for rows of more than 1024 candidate
// blocks: scores [items, NSp], NSp <= 2048
__global__ void __launch_bounds__(256) topn_cta_kernel(const float* __restrict__ pscore, int T, int G, int NSp,
                                                       int n, int lp, int fi, int fl, int32_t* __restrict__ idx) {
    __shared__ int sm[2 * 8 * 32];
    const long long item = blockIdx.x;
    const int t = (int)((item / G) % T);
    topn_row_cta_redux<256>(pscore + item * NSp, t, n, lp, fi, fl, idx + item * n, sm);
}

// one warp per (batch, token, group) item; scores [items, NSp]; NSp <= 32*PL
template <int PL>
__global__ void __launch_bounds__(256, PL <= 32 ? 3 : 1)
    topn_kernel(const float* __restrict__ pscore, long long items, int T, int G, int NSp, int n,
                int lp, int fi, int fl, int32_t* __restrict__ idx) {
    __shared__ unsigned long long wbuf[8][32];
    const int lane = threadIdx.x & 31;
    const long long item = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (item >= items) return;
    const int t = items <= 0x7fffffffLL ? (int)(((unsigned)item / (unsigned)G) % (unsigned)T)
                                        : (int)((item / G) % T);
    // the fewest slots per lane that hold the row's scored candidates (warp-uniform)
    const int nsl = (t / lp - fl - fi + 32) / 32;
    const float* row = pscore + item * NSp;
    int32_t* out = idx + item * n;
    unsigned long long* wb = wbuf[threadIdx.x >> 5];
    if (PL > 8 && nsl <= 8)
        topn_row_warp<8>(row, t, n, lp, fi, fl, out, lane, wb);
    else if (PL > 16 && nsl <= 16)
        topn_row_warp<16>(row, t, n, lp, fi, fl, out, lane, wb);
    else if (PL > 32 && nsl <= 32)
        topn_row_warp<32>(row, t, n, lp, fi, fl, out, lane, wb);
    else
        topn_row_warp<PL>(row, t, n, lp, fi, fl, out, lane, wb);
}

}  // namespace nsa
