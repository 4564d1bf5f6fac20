// k_bwd_qsel.cuh -- query gradient of the selected branch on tcgen05 tensor
// cores (pages: Top-n 块选择 / 内核设计 for the group-centric block fetches;
// natively trainable design for the backward).  With the row statistics known
// (log2-domain LSE, D = g <dO, o>), for query token t and the HG heads of its
// group over the union of its selected blocks (keys u <= t):
//   dq_h = scale * sum_u dS[h,u] k_u,   dS = P (g dP - D),  dP = <dO_h, v_u>.
// One work item is (token, group), its blocks taken in pairs of 128 keys
// staged by TMA once for all heads of the group.  The products are taken
// transposed so that the 128-row side of the instruction holds keys or
// channels:
//   S^T  = K_pair Q_t^T     M = 128 keys, N = 16 heads, K = d_k
//   dP^T = V_pair dO_t^T    M = 128 keys, N = 16 heads, K = d_v
//   softmax warps (thread = key): dS in bf16 to shared memory [16 heads][128 keys]
//   dQ  += dS K_pair        M = 64 (the 16 heads in rows 0-15), N = d_k channels
//                           (the K tile read as a transposed operand), K = 128 keys:
//                           one product per 16 keys for all channels
// An M = 64 accumulator keeps row r in TMEM lane 32 (r / 16) + r % 16, so the
// heads sit in lanes 0-15 of the first lane quadrant, read by the first warp of
// the warpgroup.  Rows 16-63 of the dS operand run past its 16-row tile into
// the neighbouring shared memory; their products land in accumulator rows no
// one reads.
// A CTA walks a range of tokens of one group; two softmax warpgroups take
// alternate tokens with their own TMEM buffers, so one token's softmax
// overlaps the other's products.  K and V of a pair sit in separate rings:
// V is needed only by dP^T and is released as soon as that product is done,
// while K stays for the dQ products, so the K ring is the deeper one.
// Warp 8 stages Q_t/dO_t and the K pairs, warp 10 the V pairs (each waits
// only on its own ring), warp 9 issues the MMAs.
#pragma once
#include "nsa_dev.cuh"
#include "k_attn_packed.cuh"
#include "k_attn_sel.cuh"
#include "k_backward.cuh"
#include "k_bwd_kv.cuh"

namespace nsa {

template <int DK, int DV>
struct BqsCfg {
    static constexpr int NQB = DK / 64, NVB = DV / 64;
    static constexpr int kQ = NQB * 2048;             // Q_t: NQB boxes [16 heads][64]
    static constexpr int kO = NVB * 2048;             // dO_t
    static constexpr int kKPair = NQB * 16384;        // per box: [128 keys][64]
    static constexpr int kVPair = NVB * 16384;
    static constexpr int NK = 3;                      // K pair slots
    static constexpr int kDS = 16 * 256;              // dS [16 heads][128 keys], two 64-key atoms
    static constexpr int kOffQ = 0;                   // 2 token slots of Q_t then dO_t
    static constexpr int kOffO = kOffQ + 2 * kQ;
    static constexpr int kOffK = ((kOffO + 2 * kO + 1023) / 1024) * 1024;
    static constexpr int kOffDS = kOffK + NK * kKPair;      // [2 warpgroups][2 buffers]
    static constexpr int kOffBar = kOffDS + 4 * kDS;
    static constexpr int kOffV = kOffBar + 1024;            // V pair slots: what is left, 1..4
    static constexpr int kSmemMax = 232448;
    static constexpr int NVfit = (kSmemMax - 1024 - kOffV) / kVPair;
    static constexpr int NV = NVfit > 4 ? 4 : NVfit;
    static constexpr int kSmem = kOffV + NV * kVPair + 1024;
    static_assert(NV >= 1 && kSmem <= kSmemMax, "shared memory");
    static constexpr int kThreads = 352;
    // TMEM per warpgroup (256 columns apart): S^T buffers 0 / 16, dP^T 32 / 48, dQ 64 .. 64 + d_k
    static constexpr uint32_t kColDP = 32, kColDQ = 64;
};

struct BqsParams {
    BwdParams bp;
    int tpc;          // tokens per CTA
    int nchunks;      // token chunks per group (grid.x = G * nchunks, group-major)
};

template <int DK, int DV, int HG>
__global__ void __launch_bounds__(352, 1)
    bwd_q_sel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapO,
              const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
              const BqsParams P) {
    using Cfg = BqsCfg<DK, DV>;
    static_assert(Cfg::kColDQ + DK <= 256 && DK % 32 == 0, "dQ columns of a warpgroup");
    const BwdParams& p = P.bp;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
    uint64_t* qfull = bars + 0;     // [2] token slots
    uint64_t* qempty = bars + 2;    // [2]
    uint64_t* kfull = bars + 4;     // [NK] K pair slots
    uint64_t* kempty = bars + 8;    // [NK]
    uint64_t* vfull = bars + 12;    // [NV] V pair slots
    uint64_t* vempty = bars + 16;   // [NV]
    uint64_t* sdfull = bars + 20;   // [2 wg][2 buf]  S^T and dP^T of a pair
    uint64_t* sdfree = bars + 24;   // [2][2]
    uint64_t* dsfull = bars + 28;   // [2][2]         dS tile written
    uint64_t* dsfree = bars + 32;   // [2][2]         dS tile read by the dQ products
    uint64_t* dqfull = bars + 36;   // [2]
    uint64_t* dqfree = bars + 38;   // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 40);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 41);
    int* npairs_ring = reinterpret_cast<int*>(bars + 42);     // [8] producer -> MMA

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int g = blockIdx.x / P.nchunks, b = blockIdx.z;
    const int tb = (blockIdx.x % P.nchunks) * P.tpc;
    const int N = min(P.tpc, p.T - tb);
    if (N <= 0) return;
    const int32_t* idx_base = p.idx + ((size_t)b * p.T * p.G + g) * p.n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&qfull[s], 1);
            mbar_init(&qempty[s], 1);
            mbar_init(&dqfull[s], 1);
            mbar_init(&dqfree[s], 4);
        }
        for (int s = 0; s < Cfg::NK; ++s) {
            mbar_init(&kfull[s], 1);
            mbar_init(&kempty[s], 1);
        }
        for (int s = 0; s < Cfg::NV; ++s) {
            mbar_init(&vfull[s], 1);
            mbar_init(&vempty[s], 1);
        }
        for (int s = 0; s < 4; ++s) {
            mbar_init(&sdfull[s], 1);
            mbar_init(&sdfree[s], 4);
            mbar_init(&dsfull[s], 4);
            mbar_init(&dsfree[s], 1);
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

    // a token's selection row: up to 16 block indices, ascending, -1 padded
    auto load_row = [&](int i, int (&r)[16]) {
        const int32_t* row = idx_base + (size_t)(tb + i) * p.G * p.n;
#pragma unroll
        for (int a = 0; a < 16; ++a) r[a] = a < p.n ? __ldg(row + a) : -1;
    };
    auto pick = [](const int (&r)[16], int a) {      // r[a] without local memory
        int v = -1;
#pragma unroll
        for (int k = 0; k < 16; ++k) v = k == a ? r[k] : v;
        return v;
    };
    auto count_row = [](const int (&r)[16]) {
        int nu = 0;
#pragma unroll
        for (int a = 0; a < 16; ++a) nu += r[a] >= 0;
        return nu;
    };

    auto lane0_wait = [&](uint64_t* bar, uint32_t parity, unsigned site) -> bool {
        bool ok = true;
        if (lane == 0) ok = wait_or_abort(bar, parity, site, abort_flag);
        return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    };
    if (warp == 8) {
        // ----------------------------------------- producer: Q_t, dO_t, K pairs
        uint32_t cnt = 0;
        bool ok = true;
        for (int i = 0; i < N && ok; ++i) {
            const int qs = i & 1;
            int r[16];
            load_row(i, r);
            const int nu = count_row(r);
            if (i >= 2 && !(ok = lane0_wait(&qempty[qs], ((i - 2) >> 1) & 1, 0x601))) break;
            if (lane == 0) {
                npairs_ring[i & 7] = (nu + 1) / 2;           // read by the MMA warp after qfull
                mbar_expect_tx(&qfull[qs], Cfg::kQ + Cfg::kO);
            }
            __syncwarp();
            if (lane < Cfg::NQB)
                tma_load_4d(smem + Cfg::kOffQ + qs * Cfg::kQ + lane * 2048, &mapQ, &qfull[qs], lane * 64, g * HG,
                            tb + i, b);
            else if (lane < Cfg::NQB + Cfg::NVB)
                tma_load_4d(smem + Cfg::kOffO + qs * Cfg::kO + (lane - Cfg::NQB) * 2048, &mapO, &qfull[qs],
                            (lane - Cfg::NQB) * 64, g * HG, tb + i, b);
            for (int pp = 0; pp < (nu + 1) / 2; ++pp) {
                const int ja = pick(r, 2 * pp), jb = 2 * pp + 1 < nu ? pick(r, 2 * pp + 1) : ja;
                const int sl = cnt % Cfg::NK;
                if (cnt >= Cfg::NK && !(ok = lane0_wait(&kempty[sl], ((cnt / Cfg::NK) - 1) & 1, 0x602))) break;
                uint8_t* base = smem + Cfg::kOffK + sl * Cfg::kKPair;
                if (lane == 0) mbar_expect_tx(&kfull[sl], Cfg::kKPair);
                __syncwarp();
                // lane 2 box + half: 64 channels (box) of block ja (half 0) or jb (half 1)
                if (lane < 2 * Cfg::NQB) {
                    const int bx = lane >> 1, half = lane & 1;
                    tma_load_4d(base + bx * 16384 + half * 8192, &mapK, &kfull[sl], bx * 64, g, (half ? jb : ja) * 64, b);
                }
                ++cnt;
            }
        }
    } else if (warp == 10) {
        // ------------------------------------------------- producer: V pairs
        uint32_t cnt = 0;
        bool ok = true;
        for (int i = 0; i < N && ok; ++i) {
            int r[16];
            load_row(i, r);
            const int nu = count_row(r);
            for (int pp = 0; pp < (nu + 1) / 2; ++pp) {
                const int ja = pick(r, 2 * pp), jb = 2 * pp + 1 < nu ? pick(r, 2 * pp + 1) : ja;
                const int sl = cnt % Cfg::NV;
                if (cnt >= Cfg::NV && !(ok = lane0_wait(&vempty[sl], ((cnt / Cfg::NV) - 1) & 1, 0x60B))) break;
                uint8_t* base = smem + Cfg::kOffV + sl * Cfg::kVPair;
                if (lane == 0) mbar_expect_tx(&vfull[sl], Cfg::kVPair);
                __syncwarp();
                if (lane < 2 * Cfg::NVB) {
                    const int bx = lane >> 1, half = lane & 1;
                    tma_load_4d(base + bx * 16384 + half * 8192, &mapV, &vfull[sl], bx * 64, g, (half ? jb : ja) * 64, b);
                }
                ++cnt;
            }
        }
    } else if (warp == 9) {
        // ----------------------------------------------------------- MMA
        // Per pair: dP^T first (its V slot returns to the producer as soon as it is
        // done), S^T, then the dQ products of the previous pair, whose dS the
        // softmax has written meanwhile.  (Issuing the two streams by readiness
        // instead measured no faster: the N = 16 products keep the pipe busy.)
        if (lane == 0) {
            constexpr uint32_t id16 = idesc_bf16(128, 16);
            constexpr uint32_t idQ = idesc_bf16_bmn(64, DK);
            uint32_t ck = 0, cv = 0;      // K and V pair slots consumed
            // per (warpgroup, buffer) q: bit q of `par` = parity of its S/dP issues so far,
            // bit q of `used` = at least one issue
            uint32_t par = 0, used = 0;
            bool ok = true;
            for (int i = 0; i < N && ok; ++i) {
                const int qs = i & 1, wg = i & 1;
                const uint32_t tw = tmem + wg * 256;
                if (!(ok = wait_or_abort(&qfull[qs], (i >> 1) & 1, 0x603, abort_flag))) break;
                const int np = npairs_ring[i & 7];
                // this warpgroup's previous token has read its dQ
                if (i >= 2 && !(ok = wait_or_abort(&dqfree[wg], ((i - 2) >> 1) & 1, 0x604, abort_flag))) break;
                tc_fence_after();
                const uint32_t sQ = smem_u32(smem + Cfg::kOffQ + qs * Cfg::kQ);
                const uint32_t sO = smem_u32(smem + Cfg::kOffO + qs * Cfg::kO);
                // pair k of this warpgroup's token stream: buffers and phases counted per warpgroup
                auto dq_pair = [&](int pp, uint32_t c) -> bool {
                    const int bf = pp & 1, q = wg * 2 + bf;
                    if (!wait_or_abort(&dsfull[q], ((par >> q) & 1) ^ 1, 0x605, abort_flag)) return false;
                    tc_fence_after();
                    const uint32_t sK = smem_u32(smem + Cfg::kOffK + (c % Cfg::NK) * Cfg::kKPair);
                    const uint32_t sD = smem_u32(smem + Cfg::kOffDS + q * Cfg::kDS);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_bf16_ss(tw + Cfg::kColDQ, sdesc_sw128(sD + (kk / 4) * 2048 + (kk % 4) * 32),
                                     sdesc_sw128_mn(sK + kk * 2048, 16384, 1024), idQ, (pp > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&dsfree[q]);
                    umma_commit(&kempty[c % Cfg::NK]);
                    return true;
                };
                for (int pp = 0; pp < np && ok; ++pp) {
                    const int bf = pp & 1, q = wg * 2 + bf;
                    const int sv = cv % Cfg::NV;
                    if (!(ok = wait_or_abort(&vfull[sv], (cv / Cfg::NV) & 1, 0x606, abort_flag))) break;
                    if (((used >> q) & 1) &&
                        !(ok = wait_or_abort(&sdfree[q], ((par >> q) & 1) ^ 1, 0x607, abort_flag)))
                        break;
                    tc_fence_after();
                    const uint32_t sV = smem_u32(smem + Cfg::kOffV + sv * Cfg::kVPair);
#pragma unroll
                    for (int kk = 0; kk < DV / 16; ++kk)
                        umma_bf16_ss(tw + Cfg::kColDP + bf * 16, sdesc_sw128(sV + (kk / 4) * 16384 + (kk % 4) * 32),
                                     sdesc_sw128(sO + (kk / 4) * 2048 + (kk % 4) * 32), id16, kk > 0 ? 1u : 0u);
                    umma_commit(&vempty[sv]);
                    ++cv;
                    const int sk = ck % Cfg::NK;
                    if (!(ok = wait_or_abort(&kfull[sk], (ck / Cfg::NK) & 1, 0x60C, abort_flag))) break;
                    tc_fence_after();
                    const uint32_t sK = smem_u32(smem + Cfg::kOffK + sk * Cfg::kKPair);
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk)
                        umma_bf16_ss(tw + bf * 16, sdesc_sw128(sK + (kk / 4) * 16384 + (kk % 4) * 32),
                                     sdesc_sw128(sQ + (kk / 4) * 2048 + (kk % 4) * 32), id16, kk > 0 ? 1u : 0u);
                    umma_commit(&sdfull[q]);
                    par ^= 1u << q;
                    used |= 1u << q;
                    if (pp >= 1) ok = dq_pair(pp - 1, ck - 1);
                    ++ck;
                }
                if (ok && np > 0) ok = dq_pair(np - 1, ck - 1);
                umma_commit(&dqfull[wg]);
                umma_commit(&qempty[qs]);
            }
        }
    } else {
        // --------------------------------- softmax / epilogue (2 warpgroups)
        const int wg = warp >> 2, wq = warp & 3;
        const int kl = wq * 32 + lane;                 // key of a pair
        const uint32_t lanebase = tmem + wg * 256 + ((uint32_t)(wq * 32) << 16);
        const float c = p.scale_log2;
        bool ok = true;
        int it = 0;
        uint32_t par = 0, used = 0;                     // per buffer: parity of its pairs, any pair
        for (int i = wg; i < N && ok; i += 2, ++it) {
            const int t = tb + i;
            int r[16];
            load_row(i, r);
            const int nu = count_row(r);
            const int np = (nu + 1) / 2;
            const size_t rowbase = ((size_t)b * p.T + t) * p.H + (size_t)g * HG;
            float L[16], Dd[16], G[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) {
                const bool hv = h < HG;
                L[h] = hv ? __ldg(p.lse2 + (rowbase + h) * 3 + kBrSlc) : INFINITY;
                Dd[h] = hv ? __ldg(p.dlt + (rowbase + h) * 3 + kBrSlc) : 0.f;
                G[h] = hv ? __ldg(p.gates + (rowbase + h) * 3 + kBrSlc) : 0.f;
            }
            for (int pp = 0; pp < np; ++pp) {
                const int bf = pp & 1, q = wg * 2 + bf;
                bool w_ok = true;
                if (lane == 0) w_ok = wait_or_abort(&sdfull[q], (par >> bf) & 1, 0x608, abort_flag);
                if (!(ok = __shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0) != 0)) break;
                tc_fence_after();
                uint32_t sr[16], dr[16];
                tmem_ld16(lanebase + bf * 16, sr);
                tmem_ld16(lanebase + Cfg::kColDP + bf * 16, dr);
                tmem_wait_ld16(sr);
                tmem_wait_ld16(dr);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sdfree[q]);
                const int un = 2 * pp + (kl >> 6);
                const bool valid = un < nu && pick(r, un) * 64 + (kl & 63) <= t;
                // the dQ products of this buffer's previous pair have read its dS tile
                if ((used >> bf) & 1) {
                    w_ok = true;
                    if (lane == 0) w_ok = wait_or_abort(&dsfree[q], ((par >> bf) & 1) ^ 1, 0x609, abort_flag);
                    if (!(ok = __shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0) != 0)) break;
                }
                const uint32_t tile = smem_u32(smem + Cfg::kOffDS + q * Cfg::kDS) + (kl >> 6) * 2048;
                const int kk = kl & 63;
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    float ds = 0.f;
                    if (valid && h < HG) {
                        const float pr = ex2a(fmaf(__uint_as_float(sr[h]), c, -L[h]));
                        ds = pr * fmaf(G[h], __uint_as_float(dr[h]), -Dd[h]);
                    }
                    __nv_bfloat16 e = __float2bfloat16_rn(ds);
                    st_shared_u16(tile + sw128_off(h, kk >> 3) + (kk & 7) * 2, *reinterpret_cast<uint16_t*>(&e));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dsfull[q]);
                par ^= 1u << bf;
                used |= 1u << bf;
            }
            // epilogue: the first warp of the warpgroup, lane = head, columns = channels
            bool w_ok = true;
            if (lane == 0) w_ok = ok && wait_or_abort(&dqfull[wg], it & 1, 0x60A, abort_flag);
            if (!(ok = __shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0) != 0)) break;
            tc_fence_after();
            if (wq == 0) {
                float* dst = p.dq + (rowbase + (lane < HG ? lane : 0)) * DK;
#pragma unroll 1
                for (int c0 = 0; c0 < DK; c0 += 32) {
                    uint32_t rq[32];
                    tmem_ld32(lanebase + Cfg::kColDQ + c0, rq);
                    tmem_wait_ld32(rq);
                    if (np > 0 && lane < HG) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            red_add_v4(dst + c0 + e, p.scale * __uint_as_float(rq[e]),
                                       p.scale * __uint_as_float(rq[e + 1]), p.scale * __uint_as_float(rq[e + 2]),
                                       p.scale * __uint_as_float(rq[e + 3]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&dqfree[wg]);
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
