// k_bwd_q.cuh -- query gradient of the compressed and window branches on
// tcgen05 tensor cores (pages: natively trainable design; 效率分析 training
// speed).  With the row statistics known (log2-domain LSE, D = g <dO, o>):
//   dq_r = scale * sum over the keys u the row sees of dS[r,u] k_u,
//   dS = P (g dP - D),  P = exp2(scale log2e q.k - LSE2),  dP = <dO_r, v_u>.
// One CTA owns a query tile of 128 rows (128/HG tokens x HG heads of one GQA
// group, the packed layout of the forward) and walks its keys in tiles of 64:
//   S  = Q K^T    M = 128 rows, N = 64 keys, K = d_k   (TMEM, 2 buffers)
//   dP = dO V^T   M = 128 rows, N = 64 keys, K = d_v   (TMEM, 2 buffers)
//   softmax warps (thread = row): dS in bf16 over S columns already read
//   dQ += dS K    M = 128 rows, N = d_k, K = 64 keys   (A from tensor memory,
//                 K as a transposed operand from the tile S read K-major)
// Keys: the window's last w tokens, or the compressed blocks complete at t.
// dq rows are disjoint between CTAs; the result is added into dq (fp32).
// Warps 0-7 softmax and epilogue (two per TMEM lane quadrant, each half of a
// key tile), warp 8 TMA, warp 9 MMA and TMEM owner.
#pragma once
#include "nsa_dev.cuh"
#include "k_attn_packed.cuh"
#include "k_backward.cuh"
#include "k_bwd_kv.cuh"

namespace nsa {

template <int DK, int DV>
struct BqCfg {
    static constexpr int NQB = DK / 64, NVB = DV / 64;
    static constexpr int kQTile = 128 * DK * 2;      // NQB boxes [128 rows][64]
    static constexpr int kOTile = 128 * DV * 2;
    static constexpr int kKT = 64 * DK * 2;          // NQB boxes [64 keys][64]
    static constexpr int kVT = 64 * DV * 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffO = kOffQ + kQTile;
    static constexpr int NSLOT = 3;                  // key tiles in flight
    static constexpr int kOffK = kOffO + kOTile;
    static constexpr int kOffV = kOffK + NSLOT * kKT;
    static constexpr int kOffBar = kOffV + NSLOT * kVT;
    static constexpr int kSmem = kOffBar + 256 + 1024;
    static_assert(kSmem <= 232448, "shared memory");
    static constexpr int kThreads = 320;
    // TMEM: S buffers 0 / 64, dP buffers 128 / 192, dQ 256
    static constexpr uint32_t kColDP = 128, kColDQ = 256;
    static_assert(kColDQ + DK <= 512, "tensor memory");
};

template <int DK, int DV, int HG, int BR>
__global__ void __launch_bounds__(320, 1)
    bwd_q_dense(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapO,
                const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                const BwdParams p) {
    using Cfg = BqCfg<DK, DV>;
    constexpr int TOK = 128 / HG;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const int b = blockIdx.z / p.G, g = blockIdx.z % p.G;
    const int t0 = blockIdx.x * TOK;
    const int t_last = min(t0 + TOK, p.T) - 1;
    // keys of the tile's rows: [k_lo, k_hi), walked in tiles of 64 from a multiple of 64
    int k_lo, k_hi;
    if (BR == kBrWin) {
        k_lo = max(0, t0 - p.w + 1) & ~63;
        k_hi = t_last + 1;
    } else {
        k_lo = 0;
        k_hi = (t_last + 1 >= p.l) ? (t_last + 1 - p.l) / p.d + 1 : 0;
    }
    const int ntiles = k_hi > k_lo ? (k_hi - k_lo + 63) / 64 : 0;
    if (ntiles == 0) return;                    // no row of the tile sees a key of this branch

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
    uint64_t* qfull = bars + 0;
    uint64_t* kvfull = bars + 1;    // [NSLOT] key tile slots
    uint64_t* kvempty = bars + 4;   // [NSLOT]
    uint64_t* sfull = bars + 7;     // [2]  S and dP of a tile (TMEM buffer j & 1)
    uint64_t* dpfree = bars + 9;    // [2]
    uint64_t* pfull = bars + 11;    // [2]  dS written
    uint64_t* dqdone = bars + 13;   // [2]  dQ product of a tile complete (S buffer free)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 16);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        mbar_init(qfull, 1);
        for (int s = 0; s < Cfg::NSLOT; ++s) {
            mbar_init(&kvfull[s], 1);
            mbar_init(&kvempty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sfull[s], 1);
            mbar_init(&dpfree[s], 8);
            mbar_init(&pfull[s], 8);
            mbar_init(&dqdone[s], 1);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ------------------------------------------------------------ TMA
        auto lane0_wait = [&](uint64_t* bar, uint32_t parity, unsigned site) -> bool {
            bool ok = true;
            if (lane == 0) ok = wait_or_abort(bar, parity, site, abort_flag);
            return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        };
        if (lane == 0) mbar_expect_tx(qfull, Cfg::kQTile + Cfg::kOTile);
        __syncwarp();
        if (lane < Cfg::NQB)
            tma_load_4d(smem + Cfg::kOffQ + lane * 16384, &mapQ, qfull, lane * 64, g * HG, t0, b);
        else if (lane < Cfg::NQB + Cfg::NVB)
            tma_load_4d(smem + Cfg::kOffO + (lane - Cfg::NQB) * 16384, &mapO, qfull, (lane - Cfg::NQB) * 64,
                        g * HG, t0, b);
        for (int j = 0; j < ntiles; ++j) {
            const int sl = j % Cfg::NSLOT;
            if (j >= Cfg::NSLOT && !lane0_wait(&kvempty[sl], ((j / Cfg::NSLOT) - 1) & 1, 0x501)) break;
            const int kb = k_lo + j * 64;
            if (lane == 0) mbar_expect_tx(&kvfull[sl], Cfg::kKT + Cfg::kVT);
            __syncwarp();
            if (lane < Cfg::NQB)
                tma_load_4d(smem + Cfg::kOffK + sl * Cfg::kKT + lane * 8192, &mapK, &kvfull[sl], lane * 64, g, kb, b);
            else if (lane < Cfg::NQB + Cfg::NVB)
                tma_load_4d(smem + Cfg::kOffV + sl * Cfg::kVT + (lane - Cfg::NQB) * 8192, &mapV, &kvfull[sl],
                            (lane - Cfg::NQB) * 64, g, kb, b);
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 64);
            constexpr uint32_t idQ = idesc_bf16_bmn(128, DK);
            const uint32_t sQ = smem_u32(smem + Cfg::kOffQ), sO = smem_u32(smem + Cfg::kOffO);
            bool ok = wait_or_abort(qfull, 0, 0x502, abort_flag);
            // Two streams: S/dP of tile js (its keys staged, its TMEM buffers free) and the
            // dQ product of tile jq (its dS written), each issued as soon as it is ready.
            int js = 0, jq = 0;
            unsigned long long t_idle = 0;
            uint32_t spins = 0;
            while (ok && jq < ntiles) {
                bool progressed = false;
                if (js < ntiles) {
                    const int sl = js % Cfg::NSLOT, bf = js & 1;
                    // S(js) overwrites the buffer whose dS fed dQ(js-2); dP(js) the one softmax(js-2) read
                    const bool ready = mbar_test_wait(&kvfull[sl], (js / Cfg::NSLOT) & 1) &&
                                       (js < 2 || (mbar_test_wait(&dqdone[bf], ((js - 2) >> 1) & 1) &&
                                                   mbar_test_wait(&dpfree[bf], ((js - 2) >> 1) & 1)));
                    if (ready) {
                        tc_fence_after();
                        const uint32_t sK = smem_u32(smem + Cfg::kOffK + sl * Cfg::kKT);
                        const uint32_t sV = smem_u32(smem + Cfg::kOffV + sl * Cfg::kVT);
#pragma unroll
                        for (int kk = 0; kk < DK / 16; ++kk)
                            umma_bf16_ss(tmem + bf * 64, sdesc_sw128(sQ + (kk / 4) * 16384 + (kk % 4) * 32),
                                         sdesc_sw128(sK + (kk / 4) * 8192 + (kk % 4) * 32), idS, kk > 0 ? 1u : 0u);
#pragma unroll
                        for (int kk = 0; kk < DV / 16; ++kk)
                            umma_bf16_ss(tmem + Cfg::kColDP + bf * 64, sdesc_sw128(sO + (kk / 4) * 16384 + (kk % 4) * 32),
                                         sdesc_sw128(sV + (kk / 4) * 8192 + (kk % 4) * 32), idS, kk > 0 ? 1u : 0u);
                        umma_commit(&sfull[bf]);
                        ++js;
                        progressed = true;
                    }
                }
                if (jq < js && mbar_test_wait(&pfull[jq & 1], (jq >> 1) & 1)) {   // dQ += dS(jq) K(jq)
                    const int sl = jq % Cfg::NSLOT, bf = jq & 1;
                    tc_fence_after();
                    const uint32_t sK = smem_u32(smem + Cfg::kOffK + sl * Cfg::kKT);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)  // keys 16kk.. : packed by warp kk / 2 in its own columns
                        umma_bf16_ts(tmem + Cfg::kColDQ, tmem + bf * 64 + (kk >> 1) * 32 + (kk & 1) * 8,
                                     sdesc_sw128_mn(sK + kk * 2048, 8192, 1024), idQ, (jq > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&dqdone[bf]);
                    umma_commit(&kvempty[sl]);
                    ++jq;
                    progressed = true;
                }
                // bounded: no progress for the wait limit ends the CTA with an error
                if (progressed) {
                    spins = 0;
                    t_idle = 0;
                } else if ((++spins & 63u) == 0u) {
                    if (*abort_flag) {
                        ok = false;
                    } else {
                        const unsigned long long now = globaltimer_ns();
                        if (t_idle == 0) t_idle = now;
                        else if (now - t_idle > kWaitLimitNs) {
                            record_timeout(0x503);
                            *abort_flag = 1;
                            ok = false;
                        }
                    }
                }
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------- softmax, epilogue
        // warp w: rows 32 (w % 4) .. +31 (its TMEM lane quadrant), keys 32 (w / 4)
        // .. +31 of each key tile
        const int quad = warp & 3, hc = warp >> 2;
        const int r = quad * 32 + lane;                  // row = TMEM lane
        const int t = t0 + r / HG, h = g * HG + r % HG;
        const bool row_ok = t < p.T;
        const size_t row = ((size_t)b * p.T + (row_ok ? t : 0)) * p.H + h;
        const float L = row_ok ? p.lse2[row * 3 + BR] : INFINITY;
        const float Dr = row_ok ? p.dlt[row * 3 + BR] : 0.f;
        const float gr = row_ok ? p.gates[row * 3 + BR] : 0.f;
        int vis_lo, vis_hi;                              // keys [vis_lo, vis_hi) of this row
        if (BR == kBrWin) {
            vis_lo = t - p.w + 1;
            vis_hi = t + 1;
        } else {
            vis_lo = 0;
            vis_hi = (t + 1 >= p.l) ? (t + 1 - p.l) / p.d + 1 : 0;
        }
        if (!row_ok || L == -INFINITY) vis_lo = vis_hi = 0;
        const uint32_t lanebase = tmem + ((uint32_t)(quad * 32) << 16);
        const float c = p.scale_log2;
        bool ok = true;
        for (int j = 0; j < ntiles; ++j) {
            const int sl = j & 1;
            bool w_ok = true;
            if (lane == 0) w_ok = wait_or_abort(&sfull[sl], (j >> 1) & 1, 0x507, abort_flag);
            if (!(ok = __shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0) != 0)) break;
            tc_fence_after();
            const int kb = k_lo + j * 64 + hc * 32;
            uint32_t sr[32], dr[32];
            tmem_ld32(lanebase + sl * 64 + hc * 32, sr);
            tmem_ld32(lanebase + Cfg::kColDP + sl * 64 + hc * 32, dr);
            tmem_wait_ld32(sr);
            tmem_wait_ld32(dr);
            uint32_t ds[16];
            // the whole key range of the tile inside the row's: no masks
            const bool inner = kb >= vis_lo && kb + 32 <= vis_hi;
#pragma unroll
            for (int cp = 0; cp < 16; ++cp) {
                float v2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int key = kb + 2 * cp + e;
                    const bool vis = inner || (key >= vis_lo && key < vis_hi);
                    const float pr = vis ? ex2a(fmaf(__uint_as_float(sr[2 * cp + e]), c, -L)) : 0.f;
                    v2[e] = pr * fmaf(gr, __uint_as_float(dr[2 * cp + e]), -Dr);
                }
                ds[cp] = pack_bf16x2(v2[0], v2[1]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&dpfree[sl]);
            // dS (bf16 pairs) over the first 16 of the 32 S columns this warp read (the
            // other warp of the quadrant may still be reading its own): the A operand
            // of dQ += dS K, read from tensor memory
            tmem_st16(lanebase + sl * 64 + hc * 32, ds);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pfull[sl]);
        }
        // epilogue: scale * dQ added into dq (columns split between the two warps of a quadrant)
        bool w_ok = true;
        const int last = ntiles - 1;
        if (lane == 0) w_ok = ok && wait_or_abort(&dqdone[last & 1], (last >> 1) & 1, 0x508, abort_flag);
        if (__shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0) != 0) {
            tc_fence_after();
            float* dst = p.dq + row * DK;
            constexpr int HALF = DK / 2;
#pragma unroll 1
            for (int c0 = hc * HALF; c0 < (hc + 1) * HALF; c0 += 32) {
                uint32_t rq[32];
                tmem_ld32(lanebase + Cfg::kColDQ + c0, rq);
                tmem_wait_ld32(rq);
                if (row_ok) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        red_add_v4(dst + c0 + e, p.scale * __uint_as_float(rq[e]), p.scale * __uint_as_float(rq[e + 1]),
                                   p.scale * __uint_as_float(rq[e + 2]), p.scale * __uint_as_float(rq[e + 3]));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace nsa
