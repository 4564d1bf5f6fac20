// k_attn_sel.cuh -- selected-block attention (page "硬件对齐+原生训练！DeepSeek NSA
// 打造高效稀疏Attention", Top-n 块选择 and 内核设计).
//
// Group-centric: one work item is (token t, GQA group g).  All HG query heads
// of the group share the selected blocks' keys/values, which are fetched once
// per item as contiguous 64-token blocks by TMA.  With only HG <= 16 query
// rows per item the products are taken transposed so that the 128-row side
// of the tensor-core instruction is filled by keys / value channels:
//   S^T = K_pair Q_t^T    M = 128 keys (two selection blocks), N = 16, K = DK
//   O^T = V^T P^T         M = 128 value channels, N = 16, K = 128 keys/pair
// One softmax runs over the union of the selected blocks' tokens u <= t.
// out[t, h] += g_slc * O / l;  lse[..., 1] = natural-log LSE.
//
// A CTA walks a range of tokens of one group (CTAs ordered group-major so a
// group's keys/values stay in L2).  Warp 8 streams Q_t and the K/V block
// pairs through a ring; warp 9 issues the MMAs in the skewed order
// S(0) S(1) O(0) S(2) O(1) ...; two softmax warpgroups (warps 0-3 and 4-7)
// take alternate tokens, each with its own S^T / O^T TMEM buffers and P^T
// tile, so one group's softmax and epilogue overlap the other's.  In a
// softmax warpgroup thread = key of a pair for S^T, value channel for O^T.
#pragma once
#include "nsa_dev.cuh"
#include "k_attn_packed.cuh"

namespace nsa {

struct SelParams {
    int B, T, H, G;
    int n;                      // selected blocks per token (<= 16), block = 64 tokens
    float scale_log2;
    const int32_t* idx;         // [B,T,G,n]
    const float* gates;         // [B,T,H,3]
    float* out;                 // [B,T,H,DV] accumulated
    float* obranch;             // [B,T,H,DV] the branch's own output o_slc (before the gate), or null
    float* lse_user;            // [B,T,H,3] or null
    int tpc;                    // tokens per CTA
    int nchunks;                // token chunks per group: grid.x = G * nchunks, group-major
};

template <int DK, int DV>
struct SelCfg {
    static constexpr int NQB = DK / 64;
    static constexpr int DVM = 128;                       // rows of the V^T operand (padded)
    static constexpr int kQSlot = NQB * 2048;             // 16 rows x 128 B per box
    static constexpr int kKPair = NQB * 16384;            // per chunk: 128 rows x 128 B
    static constexpr int kVPair = 2 * DVM * 128;
    static constexpr int kSlot = kKPair > kVPair ? kKPair : kVPair;
    static constexpr int NSLOT = 3;
    static constexpr int kOffQ = 0;
    static constexpr int kOffKV = ((2 * kQSlot + 1023) / 1024) * 1024;
    static constexpr int kOffP = kOffKV + NSLOT * kSlot;
    static constexpr int kPBytes = 16 * 2048;             // 16 heads x 1024 keys
    static constexpr int kOffRed = kOffP + 2 * kPBytes;   // one P^T tile per warpgroup
    static constexpr int kRedBytes = 2 * (2 * 4 * 16 * 4 + 2 * 16 * 4);
    static constexpr int kOffBar = kOffRed + kRedBytes;
    static constexpr int kSmem = kOffBar + 256 + 1024;
    static constexpr int kThreads = 320;
};

// order-preserving map of fp32 to u32 (for integer max reductions)
__device__ __forceinline__ uint32_t f2ord(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord2f(uint32_t u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

__device__ __forceinline__ int count_units(const int32_t* row, int n) {
    int nu = 0;
    for (int a = 0; a < n; ++a) nu += row[a] >= 0;
    return nu;
}

template <int DK, int DV, int HG>
__global__ void __launch_bounds__(320, 1)
    attn_sel_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                    const __grid_constant__ CUtensorMap mapV, const SelParams p) {
    using Cfg = SelCfg<DK, DV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
    uint64_t* qfull = bars + 0;    // [2]  per token parity
    uint64_t* qempty = bars + 2;   // [2]
    uint64_t* full = bars + 4;     // [NSLOT]
    uint64_t* empty = bars + 7;    // [NSLOT]
    uint64_t* sfull = bars + 10;   // [2]  per warpgroup
    uint64_t* sfree = bars + 12;   // [2]
    uint64_t* pfull = bars + 14;   // [2]
    uint64_t* ofull = bars + 16;   // [2]
    uint64_t* ofree = bars + 18;   // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 20);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 21);
    int* npairs_ring = reinterpret_cast<int*>(bars + 22);   // [4] producer -> MMA

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int g = blockIdx.x / p.nchunks, b = blockIdx.z;
    const int tb = (blockIdx.x % p.nchunks) * p.tpc;
    const int N = min(p.tpc, p.T - tb);

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&qfull[s], 1);
            mbar_init(&qempty[s], 1);
            mbar_init(&sfull[s], 1);
            mbar_init(&sfree[s], 4);
            mbar_init(&pfull[s], 128);
            mbar_init(&ofull[s], 1);
            mbar_init(&ofree[s], 4);
        }
        for (int s = 0; s < Cfg::NSLOT; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
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
    const int32_t* idx_base = p.idx + ((size_t)b * p.T * p.G + g) * p.n;

    if (warp == 8) {
        // ------------------------------------------------------ producer
        // The whole warp runs the loop: lane 0 waits for a free slot and posts the
        // slot's byte count, then the slot's boxes are issued from separate lanes
        // (one issuing thread alone cannot keep the TMA unit busy).
        if (N > 0) {
            if (lane == 0) {
                tma_prefetch_desc(&mapQ);
                tma_prefetch_desc(&mapK);
                tma_prefetch_desc(&mapV);
            }
            uint32_t cnt = 0;
            // warp-collective: lane 0 waits, every lane gets the outcome
            auto lane0_wait = [&](uint64_t* bar, uint32_t parity, unsigned site) -> bool {
                bool ok = true;
                if (lane == 0) ok = wait_or_abort(bar, parity, site, abort_flag);
                return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            };
            auto slot_acquire = [&](uint32_t c) -> uint8_t* {
                const int sl = c % Cfg::NSLOT;
                if (c >= Cfg::NSLOT && !lane0_wait(&empty[sl], ((c / Cfg::NSLOT) - 1) & 1, 0x301))
                    return nullptr;
                return smem + Cfg::kOffKV + sl * Cfg::kSlot;
            };
            // a token's selection row: 16 ints (ascending, -1 padded) in four
            // 16-byte loads; rows are read once and prefetched one token ahead
            auto load_row = [&](int i, int4 (&r)[4]) {
                if (i >= N) return;
                const int32_t* row = idx_base + (size_t)(tb + i) * p.G * p.n;
                if (p.n == 16 && (reinterpret_cast<uintptr_t>(row) & 15) == 0) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) r[q] = __ldg(reinterpret_cast<const int4*>(row) + q);
                } else {
                    int tmp[16];
#pragma unroll
                    for (int a = 0; a < 16; ++a) tmp[a] = a < p.n ? row[a] : -1;
#pragma unroll
                    for (int q = 0; q < 4; ++q) r[q] = make_int4(tmp[4 * q], tmp[4 * q + 1], tmp[4 * q + 2], tmp[4 * q + 3]);
                }
            };
            auto unit_of = [](const int4 (&r)[4], int a) -> int {
                const int4 v = r[a >> 2];
                const int k = a & 3;
                return k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
            };
            auto count_row = [&](const int4 (&r)[4]) -> int {
                int nu = 0;
#pragma unroll
                for (int q = 0; q < 4; ++q) nu += (r[q].x >= 0) + (r[q].y >= 0) + (r[q].z >= 0) + (r[q].w >= 0);
                return nu;
            };
            auto load_pairs = [&](const int4 (&r)[4], bool kv_is_k) -> bool {
                const int nu = count_row(r);
                for (int pp = 0; pp < (nu + 1) / 2; ++pp) {
                    const int ja = unit_of(r, 2 * pp);
                    const int jb = (2 * pp + 1 < nu) ? unit_of(r, 2 * pp + 1) : ja;
                    uint8_t* sl = slot_acquire(cnt);
                    if (!sl) return false;
                    uint64_t* bar = &full[cnt % Cfg::NSLOT];
                    if (lane == 0) mbar_expect_tx(bar, kv_is_k ? Cfg::kKPair : Cfg::kVPair);
                    __syncwarp();
                    if (kv_is_k) {
                        // lane 2*bx + half: 64 channels bx of block ja (half 0) or jb (half 1)
                        if (lane < 2 * Cfg::NQB) {
                            const int bx = lane >> 1, half = lane & 1;
                            tma_load_4d(sl + bx * 16384 + half * 8192, &mapK, bar, bx * 64, g,
                                        (half ? jb : ja) * 64, b);
                        }
                    } else if (lane < 2) {
                        tma_load_4d(sl + lane * (Cfg::DVM * 128), &mapV, bar, (lane ? jb : ja) * 64, 0, g, b);
                    }
                    ++cnt;
                }
                return true;
            };
            auto load_S = [&](int i, const int4 (&r)[4]) -> bool {
                const int qs = i & 1;
                if (i >= 2 && !lane0_wait(&qempty[qs], ((i - 2) >> 1) & 1, 0x302)) return false;
                if (lane == 0) {
                    npairs_ring[i & 3] = (count_row(r) + 1) / 2;      // read by the MMA warp
                    mbar_expect_tx(&qfull[qs], Cfg::kQSlot);            // (release)
                }
                __syncwarp();
                if (lane < Cfg::NQB)
                    tma_load_4d(smem + Cfg::kOffQ + qs * Cfg::kQSlot + lane * 2048, &mapQ, &qfull[qs],
                                lane * 64, g * HG, tb + i, b);
                return load_pairs(r, true);
            };
            int4 cur[4], prev[4], nxt[4];
            load_row(0, cur);
            load_row(1, nxt);
            bool ok = load_S(0, cur);
            for (int i = 1; i < N && ok; ++i) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    prev[q] = cur[q];
                    cur[q] = nxt[q];
                }
                load_row(i + 1, nxt);                                  // in flight during token i
                ok = load_S(i, cur);
                if (ok) ok = load_pairs(prev, false);
            }
            if (ok) load_pairs(cur, false);
        }
    } else if (warp == 9) {
        // ----------------------------------------------------------- MMA
        if (lane == 0 && N > 0) {
            constexpr uint32_t id16 = idesc_bf16(128, 16);
            uint32_t cnt = 0;
            int np_even = 0, np_odd = 0;   // pair counts of the last even / odd token (registers)
            auto slot_wait = [&](uint32_t c) -> uint32_t {
                const int sl = c % Cfg::NSLOT;
                if (!wait_or_abort(&full[sl], (c / Cfg::NSLOT) & 1, 0x303, abort_flag)) return 0;
                tc_fence_after();
                return smem_u32(smem + Cfg::kOffKV + sl * Cfg::kSlot);
            };
            auto do_S = [&](int i) -> bool {
                const int qs = i & 1, wg = i & 1;
                if (!wait_or_abort(&qfull[qs], (i >> 1) & 1, 0x304, abort_flag)) return false;
                const int np = npairs_ring[i & 3];
                if (i & 1) np_odd = np;
                else np_even = np;
                if (i >= 2 && !wait_or_abort(&sfree[wg], ((i - 2) >> 1) & 1, 0x305, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t sQ = smem_u32(smem + Cfg::kOffQ + qs * Cfg::kQSlot);
                for (int pp = 0; pp < np; ++pp) {
                    const uint32_t sK = slot_wait(cnt);
                    if (!sK) return false;
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk)
                        umma_bf16_ss(tmem + wg * 128 + pp * 16,
                                     sdesc_sw128(sK + (kk / 4) * 16384 + (kk % 4) * 32),
                                     sdesc_sw128(sQ + (kk / 4) * 2048 + (kk % 4) * 32), id16,
                                     kk > 0 ? 1u : 0u);
                    umma_commit(&empty[cnt % Cfg::NSLOT]);
                    ++cnt;
                }
                umma_commit(&sfull[wg]);
                umma_commit(&qempty[qs]);
                return true;
            };
            auto do_O = [&](int i) -> bool {
                const int wg = i & 1;
                if (!wait_or_abort(&pfull[wg], (i >> 1) & 1, 0x306, abort_flag)) return false;
                if (i >= 2 && !wait_or_abort(&ofree[wg], ((i - 2) >> 1) & 1, 0x307, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t sP = smem_u32(smem + Cfg::kOffP + wg * Cfg::kPBytes);
                const int np = (i & 1) ? np_odd : np_even;
                for (int pp = 0; pp < np; ++pp) {
                    const uint32_t sV = slot_wait(cnt);
                    if (!sV) return false;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_bf16_ss(tmem + 256 + wg * 16,
                                     sdesc_sw128(sV + (kk / 4) * (Cfg::DVM * 128) + (kk % 4) * 32),
                                     sdesc_sw128(sP + (2 * pp + kk / 4) * 2048 + (kk % 4) * 32),
                                     id16, (pp > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[cnt % Cfg::NSLOT]);
                    ++cnt;
                }
                umma_commit(&ofull[wg]);
                return true;
            };
            bool ok = do_S(0);
            for (int i = 1; i < N && ok; ++i) {
                ok = do_S(i);
                if (ok) ok = do_O(i - 1);
            }
            if (ok) do_O(N - 1);
        }
    } else {
        // ------------------------------------- softmax / epilogue (2 groups)
        const int wg = warp >> 2;                 // warpgroup: tokens i with i % 2 == wg
        const int wq = warp & 3;                  // TMEM lane quadrant
        const int kl = wq * 32 + lane;            // key within a pair / value channel
        const int unit_off = kl >> 6, tok_off = kl & 63;
        const uint32_t lanebase = tmem + ((uint32_t)(wq * 32) << 16);
        const uint32_t sP = smem_u32(smem + Cfg::kOffP + wg * Cfg::kPBytes);
        float* redm = reinterpret_cast<float*>(smem + Cfg::kOffRed + wg * (Cfg::kRedBytes / 2));
        float* redl = redm + 64;
        int* su = reinterpret_cast<int*>(redl + 64);          // [16] block ids of the token
        float* sg = redl + 80;                                 // [16] the token's selected-branch gates
        const uint32_t bar_id = 1 + wg;
        bool ok = true;
        int it = 0;
        // the token's selection entry (threads kl < 16) and gates, prefetched
        // one token ahead so their latency overlaps the previous token
        int idx_nx = -1;
        float gate_nx = 0.f;
        auto prefetch = [&](int i) {
            if (i >= N) return;
            const int32_t* row = idx_base + (size_t)(tb + i) * p.G * p.n;
            if (kl < 16) idx_nx = kl < p.n ? __ldg(row + kl) : -1;
            const size_t rb2 = ((size_t)b * p.T + tb + i) * p.H + (size_t)g * HG;
            if (kl < HG) gate_nx = __ldg(p.gates + (rb2 + kl) * 3 + 1);
            // the token's out rows (HG x DV fp32, contiguous), read-modify-written
            // by the epilogue: brought into L2 now, two tokens ahead
            if (kl * 32 < HG * DV)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(p.out + rb2 * DV + kl * 32));
        };
        prefetch(wg);
        for (int i = wg; i < N; i += 2, ++it) {
            const int t = tb + i;
            if (kl < 16) {
                su[kl] = idx_nx;
                sg[kl] = gate_nx;
            }
            const size_t rowbase = ((size_t)b * p.T + t) * p.H + (size_t)g * HG;
            named_bar_sync(bar_id, 128);
            prefetch(i + 2);
            int nu = 0;
#pragma unroll
            for (int a = 0; a < 16; ++a) nu += su[a] >= 0;
            const int npairs = (nu + 1) / 2;
            if (ok) ok = wait_or_abort(&sfull[wg], it & 1, 0x308, abort_flag);
            tc_fence_after();
            // pass A: per-head max over the valid keys
            float mx[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) mx[h] = -INFINITY;
            for (int pp = 0; pp < npairs; ++pp) {
                uint32_t r[16];
                tmem_ld16(lanebase + wg * 128 + pp * 16, r);
                tmem_wait_ld16(r);
                const int un = 2 * pp + unit_off;
                const bool valid = un < nu && su[un] * 64 + tok_off <= t;
                if (valid) {
#pragma unroll
                    for (int h = 0; h < 16; ++h) mx[h] = fmaxf(mx[h], __uint_as_float(r[h]));
                }
            }
#pragma unroll
            for (int h = 0; h < HG; ++h) {
                const uint32_t m = __reduce_max_sync(0xffffffffu, f2ord(mx[h]));
                if (lane == 0) redm[wq * 16 + h] = ord2f(m);
            }
            named_bar_sync(bar_id, 128);
#pragma unroll
            for (int h = 0; h < HG; ++h)
                mx[h] = fmaxf(fmaxf(redm[h], redm[16 + h]), fmaxf(redm[32 + h], redm[48 + h])) * p.scale_log2;
            // pass B: P = exp2(s - m), P^T to shared memory (bf16), per-head sums
            float ls[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) ls[h] = 0.f;
            for (int pp = 0; pp < npairs; ++pp) {
                uint32_t r[16];
                tmem_ld16(lanebase + wg * 128 + pp * 16, r);
                tmem_wait_ld16(r);
                const int un = 2 * pp + unit_off;
                const bool valid = un < nu && su[un] * 64 + tok_off <= t;
                const int key = pp * 128 + kl;
                const uint32_t cbase = sP + (key >> 6) * 2048;
                const int kk = key & 63;
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    float e = 0.f;
                    if (h < HG && valid) e = ex2a(fmaf(__uint_as_float(r[h]), p.scale_log2, -mx[h]));
                    ls[h] += e;
                    __nv_bfloat16 eb = __float2bfloat16_rn(e);
                    st_shared_u16(cbase + sw128_off(h, kk >> 3) + (kk & 7) * 2,
                                  *reinterpret_cast<uint16_t*>(&eb));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sfree[wg]);
            fence_proxy_async_smem();
            mbar_arrive(&pfull[wg]);
            // per-head sums: reduce-scatter over the warp, then across the 4 warps
            {
                const int base = reduce_scatter_heads<16, 16>(ls, lane);   // lanes l, l^16 hold head base
                const float v = ls[0] + __shfl_xor_sync(0xffffffffu, ls[0], 16);
                if (lane < 16) redl[wq * 16 + base] = v;
            }
            named_bar_sync(bar_id, 128);
#pragma unroll
            for (int h = 0; h < HG; ++h) ls[h] = redl[h] + redl[16 + h] + redl[32 + h] + redl[48 + h];

            // O^T: lane = value channel kl, columns = heads
            if (ok) ok = wait_or_abort(&ofull[wg], it & 1, 0x309, abort_flag);
            tc_fence_after();
            uint32_t r[16];
            tmem_ld16(lanebase + 256 + wg * 16, r);
            tmem_wait_ld16(r);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ofree[wg]);
            if (ok && kl < DV) {
                float prev[HG];
#pragma unroll
                for (int h = 0; h < HG; ++h) prev[h] = p.out[(rowbase + h) * DV + kl];
#pragma unroll
                for (int h = 0; h < HG; ++h) {
                    const float o = ls[h] > 0.f ? __uint_as_float(r[h]) / ls[h] : 0.f;
                    p.out[(rowbase + h) * DV + kl] = prev[h] + sg[h] * o;
                    if (p.obranch) p.obranch[(rowbase + h) * DV + kl] = o;
                }
            }
            if (ok && p.lse_user && kl < HG) {
                float lv = -INFINITY;
#pragma unroll
                for (int h = 0; h < HG; ++h)
                    if (h == kl) lv = ls[h] > 0.f ? (mx[h] + log2f(ls[h])) * kLn2 : -INFINITY;
                p.lse_user[(rowbase + kl) * 3 + 1] = lv;
            }
            named_bar_sync(bar_id, 128);   // su / red reuse by the next token
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
