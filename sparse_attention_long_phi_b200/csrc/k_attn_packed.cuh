// k_attn_packed.cuh -- tcgen05 attention over a contiguous key range for
// query tiles packed as (128/HG tokens) x (HG heads of one GQA group).
// Three modes:
//
//   kModeLse  compressed attention, pass 1: per-row log-sum-exp of the scaled
//             logits over the visible compressed keys (explainer, compressed
//             attention 2.4: A = Q K~^T / sqrt(d_k), softmax).
//   kModeCmp  compressed attention, pass 2: with the row LSE known,
//             P = exp(S - LSE) is the exact compressed-branch probability;
//             O = P V~ needs no rescaling.  The same P feeds the selection
//             importance scores (page 2, 重要性分数计算 / shared GQA scores):
//             each row's probabilities are mapped to selection blocks with the
//             overlap weights and summed over the HG heads of the token, then
//             written to the score table [B,T,G,NSp].  out = g_cmp * O.
//   kModeWin  sliding window (page 2, 滑动窗口): keys t-w+1 .. t, online softmax
//             with lazy rescaling of the TMEM accumulator (only when a row's
//             running max grows by more than 8 in log2 units).
//             out += g_win * O / l.
//
// One CTA takes two adjacent query tiles A and B (256 rows) that read the
// same key tiles.  Warps 0-3 run the softmax and epilogue of tile A, warps
// 4-7 those of tile B (thread = query row), warp 8 is the TMA producer and
// warp 9 the MMA issuer and TMEM owner.  The window takes key tiles of 64 keys:
//   S_x = Q_x K^T (M=128, N=64, K=DK) into one of two TMEM buffers per tile,
//   O_x += P_x V  (M=128, N=DV, K=64) with P_x written as bf16 over the S
//   columns it came from and read by the MMA from tensor memory (no shared-
//   memory round trip for P); S(j+2) is issued into a buffer only once the
//   P.V product that read P(j) from it has completed, and the MMA order
//   S_A(j+1) S_B(j+1) PV_A(j) PV_B(j) lets each tile's softmax overlap the
//   other tile's products.  The compressed passes take 128 keys per tile (Q is
//   read from shared memory once per 128 keys): pass 1 with two S buffers per
//   tile (no O), pass 2 with one (S 128 + O 128 columns per tile), in the order
//   PV_A(j) S_A(j+1) PV_B(j) S_B(j+1); the softmax reads a tile in two halves of
//   64 keys.  The softmax is issue-bound, so it is
// kept to about one FFMA + one MUFU + one add per logit, and the causal /
// window masks are applied only on the key tiles that cross a row's bound.
#pragma once
#include "nsa_dev.cuh"

namespace nsa {

enum { kModeLse = 0, kModeCmp = 1, kModeWin = 2 };

struct PackedParams {
    int B, T, H, G;
    int l, d, lp, w;
    float scale_log2;          // softmax scale * log2(e)
    const float* gates;        // [B,T,H,3]
    float* out;                // [B,T,H,DV]
    float* obranch;            // [B,T,H,DV] this branch's own output o_c (before the gate), or null
    float* lse_user;           // [B,T,H,3] or null
    float* lse_cmp;            // [B,T,H] natural log (pass 1 writes, pass 2 reads)
    float* pscore;             // [B,T,G,NSp]
    int NSp;
    int n_ctas;                // query tile pairs along the token axis (two query tiles each)
};

template <int DK, int DV, int HG, int MODE>
struct PackedCfg {
    static constexpr int TOK = 128 / HG;              // tokens per query tile
    // keys per tile: 128 in the compressed passes (an N = 128 product reads Q from
    // shared memory once per 128 keys), 64 for the window.  Pass 2 keeps one S
    // buffer per query tile (S 2 x 128 + O 2 x 128 TMEM columns); the LSE pass,
    // with no O, and the window keep two.
    static constexpr int BN = MODE == kModeWin ? 64 : 128;
    static constexpr int NBUF = MODE == kModeCmp ? 1 : 2;
    static constexpr int NQB = DK / 64;
    static constexpr int kQBytes = 128 * DK * 2;      // one tile
    static constexpr int kKBox = BN * 128;            // BN rows x 128 B
    static constexpr int kKBytes = NQB * kKBox;
    static constexpr int kVBox = DV * 128;            // DV rows x 64 keys
    static constexpr int kVBytes = kVBox * (BN / 64);
    static constexpr int kPBytes = 128 * 128;         // 128 rows x 64 keys
    static constexpr int NSK = 2;
    static constexpr int NSV = MODE == kModeLse ? 0 : (MODE == kModeCmp ? 1 : 2);
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + 2 * kQBytes;
    static constexpr int kOffV = kOffK + NSK * kKBytes;
    static constexpr int kOffP = kOffV + NSV * kVBytes;
    static constexpr int kOffBar = kOffP;             // P lives in tensor memory
    static constexpr int kSmem = kOffBar + 256 + 1024;
    static_assert(kSmem <= 232448, "shared memory");
    // TMEM: S tile A [0, NBUF BN) (NBUF buffers of BN), S tile B [NBUF BN, 2 NBUF BN),
    // then O_A, O_B from column 256
    static constexpr uint32_t kTmemCols = 512;
    static constexpr int kThreads = 320;
};

// 2^x with one MUFU instruction (ex2.approx.ftz: relative error below 2^-22,
// ex2(-inf) = +0, so masked logits need no branch)
__device__ __forceinline__ float ex2a(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Reduce `N` per-row values over the HG lanes of a token (lanes differing in
// the low log2(HG) bits) and scatter: afterwards value v of this lane holds
// the group sum of index `base + v`, with base given by bits of the lane id.
template <int N, int HG>
__device__ __forceinline__ int reduce_scatter_heads(float (&x)[N], int lane) {
    int base = 0;
    int cnt = N;
#pragma unroll
    for (int m = HG / 2; m >= 1; m >>= 1) {
        const bool hi = (lane & m) != 0;
        const int half = cnt / 2;
#pragma unroll
        for (int i = 0; i < N / 2; ++i) {
            if (i < half) {
                float send = hi ? x[i] : x[i + half];
                float keep = hi ? x[i + half] : x[i];
                x[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
            }
        }
        if (hi) base += half;
        cnt = half;
    }
    return base;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, unsigned site,
                                              volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 15u) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                record_timeout(site);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

template <int DK, int DV, int HG, int MODE, int CPS, int SPB>
__global__ void __launch_bounds__(320, 1)
    attn_packed_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                       const __grid_constant__ CUtensorMap mapV, const PackedParams p) {
    using Cfg = PackedCfg<DK, DV, HG, MODE>;
    constexpr int TOK = Cfg::TOK;
    constexpr int NSK = Cfg::NSK, NSV = Cfg::NSV;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
    uint64_t* qfull = bars + 0;
    uint64_t* kfull = bars + 1;           // [3]
    uint64_t* kempty = bars + 4;          // [3]
    uint64_t* vfull = bars + 7;           // [2]
    uint64_t* vempty = bars + 9;          // [2]
    uint64_t* sfull = bars + 11;          // [tile][buf] = 11 + 2*tile + buf
    uint64_t* sfree = bars + 15;          // [tile][buf]
    uint64_t* pfull = bars + 19;          // [tile]
    uint64_t* pvdone = bars + 21;         // [tile]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 23);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 24);
    uint64_t* qempty = bars + 25;         // the item's S products have read Q (persistent)
    uint64_t* ofree = bars + 26;          // [tile] the epilogue has read O (persistent)

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    // Work items: a pair of query tiles of one (batch, group).  Pass 1 takes one item per
    // CTA, heavy tiles first; pass 2 and the window (persistent launch, one CTA per SM)
    // stride over all items so that one item's epilogue overlaps the next item's loads and
    // products.  Every role walks the same items in the same order and counts key tiles
    // across them (jbase).
    constexpr bool kPersist = MODE != kModeLse;
    struct Item {
        int g, b, t0, t_last, key0, ntiles;
    };
    const int n_items = kPersist ? p.n_ctas * p.G * p.B : 1;
    auto item_of = [&](int iter, Item& it) -> bool {
        int cta;
        if (kPersist) {
            const int i = (int)blockIdx.x + iter * (int)gridDim.x;
            if (i >= n_items) return false;
            cta = i % p.n_ctas;
            it.g = (i / p.n_ctas) % p.G;
            it.b = i / (p.n_ctas * p.G);
        } else {
            if (iter > 0) return false;
            cta = p.n_ctas - 1 - (int)blockIdx.x;
            it.g = blockIdx.y;
            it.b = blockIdx.z;
        }
        it.t0 = cta * 2 * TOK;                         // first token of tile A
        if (it.t0 >= p.T) return false;
        it.t_last = min(it.t0 + 2 * TOK, p.T) - 1;     // last token of tile B
        // key range shared by both tiles
        if (MODE == kModeWin) {
            const int klo = max(0, it.t0 - p.w + 1);
            it.key0 = (klo / 64) * 64;
            it.ntiles = (it.t_last - it.key0) / 64 + 1;
        } else {
            const int kend = (it.t_last + 1 >= p.l) ? (it.t_last + 1 - p.l) / p.d + 1 : 0;
            it.key0 = 0;
            it.ntiles = (kend + Cfg::BN - 1) / Cfg::BN;
        }
        return true;
    };
    {
        Item it0;
        if (!item_of(0, it0)) return;                  // no work: leave before any setup
    }

    if (threadIdx.x == 0) {
        mbar_init(qfull, 1);
        for (int s = 0; s < 3; ++s) {
            mbar_init(&kfull[s], 1);
            mbar_init(&kempty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&vfull[s], 1);
            mbar_init(&vempty[s], 1);
            mbar_init(&pfull[s], 128);
            mbar_init(&pvdone[s], 1);
        }
        for (int s = 0; s < 4; ++s) {
            mbar_init(&sfull[s], 1);
            mbar_init(&sfree[s], 4);
        }
        mbar_init(qempty, 1);
        mbar_init(&ofree[0], 128);
        mbar_init(&ofree[1], 128);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&mapQ);
            tma_prefetch_desc(&mapK);
            if (MODE != kModeLse) tma_prefetch_desc(&mapV);
            int jbase = 0, qi = 0;                      // key tiles and Q loads before this item
            bool ok = true;
            Item it;
            for (int iter = 0; ok && item_of(iter, it); ++iter) {
                const int g = it.g, b = it.b, t0 = it.t0, key0 = it.key0, ntiles = it.ntiles;
                if (ntiles == 0) continue;
                // the previous item's S products have read Q
                if (qi > 0 && !(ok = wait_or_abort(qempty, (qi - 1) & 1, 0x20C, abort_flag))) break;
                mbar_expect_tx(qfull, 2 * Cfg::kQBytes);
#pragma unroll
                for (int tile = 0; tile < 2; ++tile)
#pragma unroll
                    for (int bx = 0; bx < Cfg::NQB; ++bx)
                        tma_load_4d(smem + Cfg::kOffQ + tile * Cfg::kQBytes + bx * 16384, &mapQ, qfull,
                                    bx * 64, g * HG, t0 + tile * TOK, b);
                ++qi;
                for (int jt = 0; jt < ntiles; ++jt) {
                    const int kb = key0 + jt * Cfg::BN, jg = jbase + jt;
                    const int s = jg % NSK;
                    if (jg >= NSK && !(ok = wait_or_abort(&kempty[s], ((jg / NSK) - 1) & 1, 0x201, abort_flag)))
                        break;
                    uint8_t* ks = smem + Cfg::kOffK + s * Cfg::kKBytes;
                    mbar_expect_tx(&kfull[s], Cfg::kKBytes);
#pragma unroll
                    for (int bx = 0; bx < Cfg::NQB; ++bx)
#pragma unroll
                        for (int hb = 0; hb < Cfg::BN / 64; ++hb)   // boxes of 64 rows
                            tma_load_4d(ks + bx * Cfg::kKBox + hb * 8192, &mapK, &kfull[s], bx * 64, g, kb + hb * 64, b);
                    if (MODE != kModeLse) {
                        const int sv = jg % NSV;
                        if (jg >= NSV && !(ok = wait_or_abort(&vempty[sv], ((jg / NSV) - 1) & 1, 0x202, abort_flag)))
                            break;
                        uint8_t* vs = smem + Cfg::kOffV + sv * Cfg::kVBytes;
                        mbar_expect_tx(&vfull[sv], Cfg::kVBytes);
#pragma unroll
                        for (int hb = 0; hb < Cfg::BN / 64; ++hb)
                            tma_load_4d(vs + hb * Cfg::kVBox, &mapV, &vfull[sv], kb + hb * 64, 0, g, b);
                    }
                }
                jbase += ntiles;
            }
        }
    } else if (warp == 9) {
        // ----------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, Cfg::BN);
            constexpr uint32_t idO = idesc_bf16(128, DV);
            int jbase = 0, qi = 0;
            bool ok = true;
            Item it;
            for (int iter = 0; ok && item_of(iter, it); ++iter) {
                const int ntiles = it.ntiles;
                if (ntiles == 0) continue;
                if (!(ok = wait_or_abort(qfull, qi & 1, 0x203, abort_flag))) break;
                // the previous item's last P.V products have completed: its S buffers are
                // free, and every pvdone phase waited for below belongs to this item
                if (MODE != kModeLse && qi > 0)
                    for (int tile = 0; tile < 2 && ok; ++tile)
                        ok = wait_or_abort(&pvdone[tile], (jbase - 1) & 1, 0x20D, abort_flag);
                if (!ok) break;
                // S of key tile jt for query tile `tile` (and both tiles when tile < 0)
                auto issue_S = [&](int jt, int only) -> bool {
                    const int jg = jbase + jt;
                    const int s = jg % NSK, buf = Cfg::NBUF == 2 ? (jg & 1) : 0;
                    if (only <= 0 && !wait_or_abort(&kfull[s], (jg / NSK) & 1, 0x204, abort_flag)) return false;
                    const uint32_t sK = smem_u32(smem + Cfg::kOffK + s * Cfg::kKBytes);
#pragma unroll
                    for (int tile = 0; tile < 2; ++tile) {
                        if (only >= 0 && tile != only) continue;
                        if (MODE == kModeLse && jg >= 2 &&
                            !wait_or_abort(&sfree[2 * tile + buf], ((jg - 2) >> 1) & 1, 0x205, abort_flag))
                            return false;
                        // the buffer's P(jt - NBUF) must have been read by its P.V product: an
                        // MMA writing tensor memory is not ordered behind an earlier MMA that
                        // reads the same columns as its A operand
                        if (MODE != kModeLse && jt >= Cfg::NBUF &&
                            !wait_or_abort(&pvdone[tile], (jg - Cfg::NBUF) & 1, 0x20B, abort_flag))
                            return false;
                        tc_fence_after();
                        const uint32_t sQ = smem_u32(smem + Cfg::kOffQ + tile * Cfg::kQBytes);
#pragma unroll
                        for (int kk = 0; kk < DK / 16; ++kk)
                            umma_bf16_ss(tmem + tile * Cfg::NBUF * Cfg::BN + buf * Cfg::BN,
                                         sdesc_sw128(sQ + (kk / 4) * 16384 + (kk % 4) * 32),
                                         sdesc_sw128(sK + (kk / 4) * Cfg::kKBox + (kk % 4) * 32), idS,
                                         kk > 0 ? 1u : 0u);
                        umma_commit(&sfull[2 * tile + buf]);
                    }
                    if (only != 0) umma_commit(&kempty[s]);       // both tiles have read the K stage
                    // after the item's last S products the Q tiles may be replaced
                    if (only != 0 && jt == ntiles - 1) umma_commit(qempty);
                    return true;
                };
                // P.V of key tile jt for query tile `tile` (and both tiles when tile < 0)
                auto issue_PV = [&](int jt, int only) -> bool {
                    const int jg = jbase + jt;
                    const int sv = jg % NSV;
                    if (only <= 0 && !wait_or_abort(&vfull[sv], (jg / NSV) & 1, 0x207, abort_flag)) return false;
                    const uint32_t sV = smem_u32(smem + Cfg::kOffV + sv * Cfg::kVBytes);
#pragma unroll
                    for (int tile = 0; tile < 2; ++tile) {
                        if (only >= 0 && tile != only) continue;
                        if (!wait_or_abort(&pfull[tile], jg & 1, 0x206, abort_flag)) return false;
                        // the first product of an item overwrites O: the previous item's
                        // epilogue must have read it
                        if (jt == 0 && qi > 0 && !wait_or_abort(&ofree[tile], (qi - 1) & 1, 0x20E, abort_flag))
                            return false;
                        tc_fence_after();
                        // P (bf16 pairs) over the first BN/2 columns of S(jt)
                        const uint32_t tP = tmem + tile * Cfg::NBUF * Cfg::BN + (Cfg::NBUF == 2 ? (jg & 1) : 0) * Cfg::BN;
#pragma unroll
                        for (int kk = 0; kk < Cfg::BN / 16; ++kk)
                            umma_bf16_ts(tmem + 256 + tile * DV, tP + kk * 8,
                                         sdesc_sw128(sV + (kk / 4) * Cfg::kVBox + (kk % 4) * 32), idO,
                                         (jt > 0 || kk > 0) ? 1u : 0u);
                        umma_commit(&pvdone[tile]);
                    }
                    if (only != 0) umma_commit(&vempty[sv]);      // both tiles have read the V stage
                    return true;
                };
                if (Cfg::NBUF == 2) {
                    // S(jt+1) into the other buffer while the softmax works on S(jt)
                    ok = issue_S(0, -1);
                    for (int jt = 0; jt < ntiles && ok; ++jt) {
                        if (jt + 1 < ntiles) ok = issue_S(jt + 1, -1);
                        if (ok && MODE != kModeLse) ok = issue_PV(jt, -1);
                    }
                } else {
                    // one S buffer per query tile: P.V(jt) of a tile, then its S(jt+1) into
                    // the same columns; the two tiles alternate so that one tile's products
                    // run while the other's softmax does
                    ok = issue_S(0, 0);
                    if (ok) ok = issue_S(0, 1);
                    for (int jt = 0; jt < ntiles && ok; ++jt) {
                        ok = issue_PV(jt, 0);
                        if (ok && jt + 1 < ntiles) ok = issue_S(jt + 1, 0);
                        if (ok) ok = issue_PV(jt, 1);
                        if (ok && jt + 1 < ntiles) ok = issue_S(jt + 1, 1);
                    }
                }
                ++qi;
                jbase += ntiles;
            }
        }
    } else {
        // ------------------------------------------------ softmax / epilogue
        const int tile = warp >> 2;                 // 0: tile A, 1: tile B
        const int wq = warp & 3;                    // TMEM lane quadrant
        const int r = wq * 32 + lane;               // row within the tile
        int jbase = 0;                              // key tiles before this item
        Item it;
        for (int iter = 0; item_of(iter, it); ++iter) {
        const int g = it.g, b = it.b, t0 = it.t0, key0 = it.key0, ntiles = it.ntiles;
        const int t = t0 + tile * TOK + r / HG;
        const int hh = r % HG;
        const int h = g * HG + hh;
        const bool row_ok = t < p.T;
        const size_t rowid = ((size_t)b * p.T + (row_ok ? t : 0)) * p.H + h;
        const uint32_t lanebase = tmem + ((uint32_t)(wq * 32) << 16);
        const uint32_t sbase = lanebase + tile * Cfg::NBUF * Cfg::BN; // S buffers of this tile
        const uint32_t obase = lanebase + 256 + tile * DV;    // O of this tile
        int vis_hi, vis_lo = 0;
        if (MODE == kModeWin) {
            vis_hi = t + 1;
            vis_lo = t - p.w + 1;
        } else {
            vis_hi = (t + 1 >= p.l) ? (t + 1 - p.l) / p.d + 1 : 0;
        }
        if (!row_ok) vis_hi = vis_lo = -1 << 30;
        if (MODE == kModeWin && row_ok) {
            // the epilogue adds into this row of out: start bringing it into L2 now,
            // so its read does not wait on DRAM after the last key tile
            const char* orow = reinterpret_cast<const char*>(p.out + rowid * DV);
#pragma unroll
            for (int q = 0; q < DV * 4; q += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(orow + q));
        }
        // bounds shared by every row of this query tile (visibility grows with t)
        const int tile_first = t0 + tile * TOK;
        const int tile_last = min(tile_first + TOK, p.T) - 1;
        const int vis_first = (tile_first + 1 >= p.l) ? (tile_first + 1 - p.l) / p.d + 1 : 0;
        float m_run = -INFINITY, l_run = 0.f;
        float lse2 = -INFINITY;
        if (MODE == kModeCmp && row_ok) lse2 = p.lse_cmp[rowid] * kLog2e;
        constexpr int NB = 64 / SPB;                        // complete blocks per tile
        constexpr int NJ = (63 + CPS - 1) / SPB + 1;        // partial blocks touched per tile
        constexpr int NC = NJ - NB;                         // carried into the next tile
        float carry[NC > 0 ? NC : 1];
#pragma unroll
        for (int c = 0; c < (NC > 0 ? NC : 1); ++c) carry[c] = 0.f;
        bool ok = true;

        if (MODE == kModeLse) {
            // BN = 128 keys per tile, read from TMEM in two halves of 64
            for (int jt = 0; jt < ntiles; ++jt) {
                const int jg = jbase + jt, buf = jg & 1;
                if (ok) ok = wait_or_abort(&sfull[2 * tile + buf], (jg >> 1) & 1, 0x208, abort_flag);
                tc_fence_after();
#pragma unroll 1
                for (int hb = 0; hb < Cfg::BN / 64; ++hb) {
                    const int kb = key0 + jt * Cfg::BN + hb * 64;
                    uint32_t ra[32], rb[32];
                    tmem_ld32(sbase + buf * Cfg::BN + hb * 64, ra);
                    tmem_ld32(sbase + buf * Cfg::BN + hb * 64 + 32, rb);
                    tmem_wait_ld32(ra);
                    tmem_wait_ld32(rb);
                    float s[64];
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        s[k] = __uint_as_float(ra[k]);
                        s[k + 32] = __uint_as_float(rb[k]);
                    }
                    if (!(kb + 64 <= vis_first)) {
#pragma unroll
                        for (int k = 0; k < 64; ++k)
                            if (!(kb + k >= vis_lo && kb + k < vis_hi)) s[k] = -INFINITY;
                    }
                    const float c = p.scale_log2;
                    float mr = -INFINITY;
#pragma unroll
                    for (int k = 0; k < 64; ++k) mr = fmaxf(mr, s[k]);
                    const float mn = fmaxf(m_run, mr * c);
                    if (mn != -INFINITY) {
                        // even and odd columns summed separately, two per packed instruction
                        float2 acc = make_float2(0.f, 0.f);
                        const float2 c2 = make_float2(c, c), nm2 = make_float2(-mn, -mn);
#pragma unroll
                        for (int k = 0; k < 64; k += 2) {
                            const float2 a = __ffma2_rn(make_float2(s[k], s[k + 1]), c2, nm2);
                            acc = __fadd2_rn(acc, make_float2(ex2a(a.x), ex2a(a.y)));
                        }
                        l_run = l_run * ex2a(m_run - mn) + (acc.x + acc.y);
                        m_run = mn;
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfree[2 * tile + buf]);
            }
        }
        for (int jt = 0; MODE != kModeLse && jt < ntiles; ++jt) {
            const int jg = jbase + jt;
            const int buf = Cfg::NBUF == 2 ? (jg & 1) : 0;
            if (ok) ok = wait_or_abort(&sfull[2 * tile + buf], (Cfg::NBUF == 2 ? (jg >> 1) : jg) & 1, 0x208, abort_flag);
            tc_fence_after();
            // the key tile in halves of 64 keys (one half for the window)
#pragma unroll 1
            for (int hb = 0; hb < Cfg::BN / 64; ++hb) {
            const int kb = key0 + jt * Cfg::BN + hb * 64;
            uint32_t ra[32], rb[32];
            tmem_ld32(sbase + buf * Cfg::BN + hb * 64, ra);
            tmem_ld32(sbase + buf * Cfg::BN + hb * 64 + 32, rb);
            tmem_wait_ld32(ra);
            tmem_wait_ld32(rb);
            float s[64];
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                s[k] = __uint_as_float(ra[k]);
                s[k + 32] = __uint_as_float(rb[k]);
            }
            // masks only where the key tile crosses a row bound of this query tile
            const bool interior = (MODE == kModeWin)
                                      ? (kb >= tile_last - p.w + 1 && kb + 63 <= tile_first)
                                      : (kb + 64 <= vis_first);
            if (!interior) {
#pragma unroll
                for (int k = 0; k < 64; ++k) {
                    const int key = kb + k;
                    if (!(key >= vis_lo && key < vis_hi)) s[k] = -INFINITY;
                }
            }
            const float c = p.scale_log2;
            float pr[64];
            float alpha = 1.f;
            bool need_rescale = false;
            if (MODE == kModeCmp) {
                // a row with no visible key has LSE = -inf and only masked logits
                const float nl = lse2 == -INFINITY ? 0.f : -lse2;
                const float2 c2 = make_float2(c, c), nl2 = make_float2(nl, nl);
#pragma unroll
                for (int k = 0; k < 64; k += 2) {
                    const float2 a = __ffma2_rn(make_float2(s[k], s[k + 1]), c2, nl2);
                    pr[k] = ex2a(a.x);
                    pr[k + 1] = ex2a(a.y);
                }
            } else {
                float mr = -INFINITY;
#pragma unroll
                for (int k = 0; k < 64; ++k) mr = fmaxf(mr, s[k]);
                const float mt = mr * c;
                if (mt > m_run + 8.f) {
                    alpha = ex2a(m_run - mt);        // 0 when m_run = -inf
                    l_run *= alpha;
                    m_run = mt;
                    need_rescale = true;
                }
                // m_run stays -inf while every key so far is masked for this row
                const float nm = m_run == -INFINITY ? 0.f : -m_run;
                const float2 c2 = make_float2(c, c), nm2 = make_float2(nm, nm);
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < 64; k += 2) {
                    const float2 a = __ffma2_rn(make_float2(s[k], s[k + 1]), c2, nm2);
                    pr[k] = ex2a(a.x);
                    pr[k + 1] = ex2a(a.y);
                    acc = __fadd2_rn(acc, make_float2(pr[k], pr[k + 1]));
                }
                l_run += acc.x + acc.y;
            }
            if (MODE == kModeCmp) {
                // importance scores of selection blocks kb/SPB .. kb/SPB + NB - 1
                float part[NJ];
                if constexpr (SPB == 4 && CPS == 2) {
                    // key 4m+u feeds block m twice for u < 3; key 4m+3 feeds blocks m
                    // and m+1 once: part[m] = 2 (p0+p1+p2+p3) - p3 + p(4m-1), with
                    // p(-1) the last key of the previous tile (carried)
#pragma unroll
                    for (int m = 0; m < NB; ++m) {
                        const float2 q = __fadd2_rn(make_float2(pr[4 * m], pr[4 * m + 1]),
                                                    make_float2(pr[4 * m + 2], pr[4 * m + 3]));
                        const float prev = m == 0 ? carry[0] : pr[4 * m - 1];
                        part[m] = fmaf(2.f, q.x + q.y, prev - pr[4 * m + 3]);
                    }
                    carry[0] = pr[63];
                } else {
#pragma unroll
                    for (int m = 0; m < NJ; ++m) part[m] = 0.f;
#pragma unroll
                    for (int c = 0; c < NC; ++c) part[c] += carry[c];
#pragma unroll
                    for (int k = 0; k < 64; ++k)
#pragma unroll
                        for (int u = 0; u < CPS; ++u) part[(k + u) / SPB] += pr[k];
#pragma unroll
                    for (int c = 0; c < NC; ++c) carry[c] = part[NB + c];
                }
                float red[NB];
#pragma unroll
                for (int m = 0; m < NB; ++m) red[m] = part[m];
                const int base = reduce_scatter_heads<NB, HG>(red, lane);
                if (row_ok) {
                    const int j0 = kb / SPB;
                    float* dst = p.pscore + (((size_t)b * p.T + t) * p.G + g) * p.NSp;
#pragma unroll
                    for (int v = 0; v < NB / HG; ++v)
                        if (j0 + base + v < p.NSp) dst[j0 + base + v] = red[v];
                }
            }
            // the previous P.V of this tile finished: the window's O rescale needs it,
            // and it keeps this loop at most one pvdone phase ahead of the MMA warp
            // (a parity wait cannot tell phases two apart; the epilogue relies on it)
            if (hb == 0 && jt > 0 && ok) ok = wait_or_abort(&pvdone[tile], (jg - 1) & 1, 0x209, abort_flag);
            tc_fence_after();
            if (MODE == kModeWin && jt > 0 && __any_sync(0xffffffffu, need_rescale)) {
                const float a = need_rescale ? alpha : 1.f;
#pragma unroll 1
                for (int c0 = 0; c0 < DV; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(obase + c0, o);
                    tmem_wait_ld32(o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * a);
                    tmem_st32(obase + c0, o);
                }
                tmem_wait_st();
            }
            // P (bf16, two per column) over the first BN/2 columns of S(jt), 32 per
            // half: the A operand of this tile's P.V product (half 1's columns 32-63
            // held keys of half 0, already read)
            {
                uint32_t pk[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(pr[2 * c], pr[2 * c + 1]);
                tmem_st32(sbase + buf * Cfg::BN + hb * 32, pk);
                tmem_wait_st();
            }
            }
            tc_fence_before();
            mbar_arrive(&pfull[tile]);
        }

        // ------------------------------------------------------- epilogue
        if (MODE == kModeLse) {
            if (row_ok) {
                const float lse = (l_run > 0.f) ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
                p.lse_cmp[rowid] = lse;
                if (p.lse_user) p.lse_user[rowid * 3 + 0] = lse;
            }
        } else {
            if (MODE == kModeCmp && NC > 0) {
                // flush the carried partial scores of the block after the last tile
                const int jn = (key0 + ntiles * Cfg::BN) / SPB;
#pragma unroll
                for (int c = 0; c < (NC > 0 ? NC : 1); ++c) {
                    float v = carry[c];
#pragma unroll
                    for (int m = HG / 2; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
                    if (row_ok && hh == 0 && ntiles > 0 && jn + c < p.NSp)
                        p.pscore[(((size_t)b * p.T + t) * p.G + g) * p.NSp + jn + c] = v;
                }
            }
            if (ntiles > 0 && ok) ok = wait_or_abort(&pvdone[tile], (jbase + ntiles - 1) & 1, 0x20A, abort_flag);
            tc_fence_after();
            const float gate = row_ok ? p.gates[rowid * 3 + (MODE == kModeCmp ? 0 : 2)] : 0.f;
            const float inv = (MODE == kModeWin) ? (l_run > 0.f ? 1.f / l_run : 0.f) : 1.f;
#pragma unroll 1
            for (int c0 = 0; c0 < DV; c0 += 32) {
                uint32_t o[32];
                if (ntiles > 0) {
                    tmem_ld32(obase + c0, o);
                    tmem_wait_ld32(o);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = 0u;
                }
                if (row_ok && ok && p.obranch) {
                    float4* dsto = reinterpret_cast<float4*>(p.obranch + rowid * DV + c0);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dsto[e] = make_float4(__uint_as_float(o[4 * e + 0]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                                              __uint_as_float(o[4 * e + 2]) * inv, __uint_as_float(o[4 * e + 3]) * inv);
                }
                if (row_ok && ok) {
                    float4* dst = reinterpret_cast<float4*>(p.out + rowid * DV + c0);
                    float4 prev[8];
                    if (MODE == kModeWin) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) prev[e] = dst[e];
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        float4 v;
                        v.x = gate * __uint_as_float(o[4 * e + 0]) * inv;
                        v.y = gate * __uint_as_float(o[4 * e + 1]) * inv;
                        v.z = gate * __uint_as_float(o[4 * e + 2]) * inv;
                        v.w = gate * __uint_as_float(o[4 * e + 3]) * inv;
                        if (MODE == kModeWin) {
                            v.x += prev[e].x;
                            v.y += prev[e].y;
                            v.z += prev[e].z;
                            v.w += prev[e].w;
                        }
                        dst[e] = v;
                    }
                }
            }
            if (MODE == kModeWin && row_ok && p.lse_user)
                p.lse_user[rowid * 3 + 2] = (m_run + log2f(l_run)) * kLn2;
            if (ntiles > 0) {
                // this tile's O has been read: the next item's first P.V may overwrite it
                tc_fence_before();
                mbar_arrive(&ofree[tile]);
            }
        }
        jbase += ntiles;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::kTmemCols);
    }
}

}  // namespace nsa
