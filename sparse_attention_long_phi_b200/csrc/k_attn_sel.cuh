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
// A CTA walks a range of tokens of one group.  Warp 4 streams Q_t and the
// K/V block pairs through a ring; warp 5 issues MMAs in the skewed order
// S(0) S(1) O(0) S(2) O(1) ... so the next token's S^T overlaps the current
// token's softmax; warps 0-3 run the softmax (thread = key of a pair for S^T,
// value channel for O^T) and the epilogue.
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
    float* lse_user;            // [B,T,H,3] or null
    int tpc;                    // tokens per CTA
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
    static constexpr int kOffRed = kOffP + kPBytes;
    static constexpr int kOffBar = kOffRed + 2 * 4 * 16 * 4;
    static constexpr int kSmem = kOffBar + 256 + 1024;
};

__device__ __forceinline__ int load_units(const int32_t* row, int n, int (&u)[16]) {
    int nu = 0;
#pragma unroll
    for (int a = 0; a < 16; ++a) {
        int j = a < n ? row[a] : -1;
        if (j >= 0) u[nu++] = j;
    }
    return nu;
}

template <int DK, int DV>
__global__ void __launch_bounds__(192, 1)
    attn_sel_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                    const __grid_constant__ CUtensorMap mapV, const SelParams p) {
    using Cfg = SelCfg<DK, DV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
    uint64_t* qfull = bars + 0;    // [2]
    uint64_t* qempty = bars + 2;   // [2]
    uint64_t* full = bars + 4;     // [NSLOT]
    uint64_t* empty = bars + 7;    // [NSLOT]
    uint64_t* sfull = bars + 10;   // [2]
    uint64_t* sfree = bars + 12;   // [2]
    uint64_t* pfull = bars + 14;
    uint64_t* ofull = bars + 15;   // [2]
    uint64_t* ofree = bars + 17;   // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 20);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 21);
    float* redm = reinterpret_cast<float*>(smem + Cfg::kOffRed);
    float* redl = redm + 64;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int g = blockIdx.y, b = blockIdx.z;
    const int HG = p.H / p.G;
    const int tb = blockIdx.x * p.tpc;
    const int N = min(p.tpc, p.T - tb);

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&qfull[s], 1);
            mbar_init(&qempty[s], 1);
            mbar_init(&sfull[s], 1);
            mbar_init(&sfree[s], 4);
            mbar_init(&ofull[s], 1);
            mbar_init(&ofree[s], 4);
        }
        for (int s = 0; s < Cfg::NSLOT; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(pfull, 128);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int32_t* idx_base = p.idx + ((size_t)b * p.T * p.G + g) * p.n;

    if (warp == 4) {
        // ------------------------------------------------------ producer
        if (lane == 0 && N > 0) {
            tma_prefetch_desc(&mapQ);
            tma_prefetch_desc(&mapK);
            tma_prefetch_desc(&mapV);
            uint32_t cnt = 0;
            bool ok = true;
            auto slot_acquire = [&](uint32_t c) -> uint8_t* {
                const int sl = c % Cfg::NSLOT;
                if (c >= Cfg::NSLOT &&
                    !wait_or_abort(&empty[sl], ((c / Cfg::NSLOT) - 1) & 1, 0x301, abort_flag))
                    return nullptr;
                return smem + Cfg::kOffKV + sl * Cfg::kSlot;
            };
            auto load_S = [&](int i) -> bool {
                const int t = tb + i;
                const int qs = i & 1;
                if (i >= 2 && !wait_or_abort(&qempty[qs], ((i - 2) >> 1) & 1, 0x302, abort_flag))
                    return false;
                mbar_expect_tx(&qfull[qs], Cfg::kQSlot);
                for (int bx = 0; bx < Cfg::NQB; ++bx)
                    tma_load_4d(smem + Cfg::kOffQ + qs * Cfg::kQSlot + bx * 2048, &mapQ, &qfull[qs],
                                bx * 64, g * HG, t, b);
                int u[16];
                const int nu = load_units(idx_base + (size_t)t * p.G * p.n, p.n, u);
                for (int pp = 0; pp < (nu + 1) / 2; ++pp) {
                    const int ja = u[2 * pp], jb = (2 * pp + 1 < nu) ? u[2 * pp + 1] : ja;
                    uint8_t* sl = slot_acquire(cnt);
                    if (!sl) return false;
                    uint64_t* bar = &full[cnt % Cfg::NSLOT];
                    mbar_expect_tx(bar, Cfg::kKPair);
                    for (int bx = 0; bx < Cfg::NQB; ++bx) {
                        tma_load_4d(sl + bx * 16384, &mapK, bar, bx * 64, g, ja * 64, b);
                        tma_load_4d(sl + bx * 16384 + 8192, &mapK, bar, bx * 64, g, jb * 64, b);
                    }
                    ++cnt;
                }
                return true;
            };
            auto load_O = [&](int i) -> bool {
                const int t = tb + i;
                int u[16];
                const int nu = load_units(idx_base + (size_t)t * p.G * p.n, p.n, u);
                for (int pp = 0; pp < (nu + 1) / 2; ++pp) {
                    const int ja = u[2 * pp], jb = (2 * pp + 1 < nu) ? u[2 * pp + 1] : ja;
                    uint8_t* sl = slot_acquire(cnt);
                    if (!sl) return false;
                    uint64_t* bar = &full[cnt % Cfg::NSLOT];
                    mbar_expect_tx(bar, Cfg::kVPair);
                    tma_load_4d(sl, &mapV, bar, ja * 64, 0, g, b);
                    tma_load_4d(sl + Cfg::DVM * 128, &mapV, bar, jb * 64, 0, g, b);
                    ++cnt;
                }
                return true;
            };
            ok = load_S(0);
            for (int i = 1; i < N && ok; ++i) {
                ok = load_S(i);
                if (ok) ok = load_O(i - 1);
            }
            if (ok) load_O(N - 1);
        }
    } else if (warp == 5) {
        // ----------------------------------------------------------- MMA
        if (lane == 0 && N > 0) {
            constexpr uint32_t id16 = idesc_bf16(128, 16);
            uint32_t cnt = 0;
            auto slot_wait = [&](uint32_t c) -> uint32_t {
                const int sl = c % Cfg::NSLOT;
                if (!wait_or_abort(&full[sl], (c / Cfg::NSLOT) & 1, 0x303, abort_flag)) return 0;
                tc_fence_after();
                return smem_u32(smem + Cfg::kOffKV + sl * Cfg::kSlot);
            };
            auto do_S = [&](int i) -> bool {
                const int t = tb + i;
                const int qs = i & 1;
                if (!wait_or_abort(&qfull[qs], (i >> 1) & 1, 0x304, abort_flag)) return false;
                if (i >= 2 && !wait_or_abort(&sfree[qs], ((i - 2) >> 1) & 1, 0x305, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t sQ = smem_u32(smem + Cfg::kOffQ + qs * Cfg::kQSlot);
                int u[16];
                const int nu = load_units(idx_base + (size_t)t * p.G * p.n, p.n, u);
                for (int pp = 0; pp < (nu + 1) / 2; ++pp) {
                    const uint32_t sK = slot_wait(cnt);
                    if (!sK) return false;
#pragma unroll
                    for (int kk = 0; kk < DK / 16; ++kk)
                        umma_bf16_ss(tmem + qs * 128 + pp * 16,
                                     sdesc_sw128(sK + (kk / 4) * 16384 + (kk % 4) * 32),
                                     sdesc_sw128(sQ + (kk / 4) * 2048 + (kk % 4) * 32), id16,
                                     kk > 0 ? 1u : 0u);
                    umma_commit(&empty[cnt % Cfg::NSLOT]);
                    ++cnt;
                }
                umma_commit(&sfull[qs]);
                umma_commit(&qempty[qs]);
                return true;
            };
            auto do_O = [&](int i) -> bool {
                const int t = tb + i;
                const int ob = i & 1;
                if (!wait_or_abort(pfull, i & 1, 0x306, abort_flag)) return false;
                if (i >= 2 && !wait_or_abort(&ofree[ob], ((i - 2) >> 1) & 1, 0x307, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t sP = smem_u32(smem + Cfg::kOffP);
                int u[16];
                const int nu = load_units(idx_base + (size_t)t * p.G * p.n, p.n, u);
                for (int pp = 0; pp < (nu + 1) / 2; ++pp) {
                    const uint32_t sV = slot_wait(cnt);
                    if (!sV) return false;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_bf16_ss(tmem + 256 + ob * 16,
                                     sdesc_sw128(sV + (kk / 4) * (Cfg::DVM * 128) + (kk % 4) * 32),
                                     sdesc_sw128(sP + (2 * pp + kk / 4) * 2048 + (kk % 4) * 32),
                                     id16, (pp > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[cnt % Cfg::NSLOT]);
                    ++cnt;
                }
                umma_commit(&ofull[ob]);
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
        // ------------------------------------------------ softmax / epilogue
        const int kl = threadIdx.x;                  // key within a pair / value channel
        const int unit_off = kl >> 6, tok_off = kl & 63;
        const uint32_t lanebase = tmem + ((uint32_t)(warp * 32) << 16);
        const uint32_t sP = smem_u32(smem + Cfg::kOffP);
        bool ok = true;
        for (int i = 0; i < N; ++i) {
            const int t = tb + i;
            const int sb = i & 1;
            int u[16];
            const int nu = load_units(idx_base + (size_t)t * p.G * p.n, p.n, u);
            const int npairs = (nu + 1) / 2;
            if (ok) ok = wait_or_abort(&sfull[sb], (i >> 1) & 1, 0x308, abort_flag);
            tc_fence_after();
            float mx[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) mx[h] = -INFINITY;
            for (int pp = 0; pp < npairs; ++pp) {
                uint32_t r[16];
                tmem_ld16(lanebase + sb * 128 + pp * 16, r);
                tmem_wait_ld16(r);
                const int un = 2 * pp + unit_off;
                const bool valid = un < nu && (un < 16 ? (u[un] * 64 + tok_off <= t) : false);
                if (valid) {
#pragma unroll
                    for (int h = 0; h < 16; ++h) mx[h] = fmaxf(mx[h], __uint_as_float(r[h]) * p.scale_log2);
                }
            }
#pragma unroll
            for (int h = 0; h < 16; ++h) {
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], o));
            }
            if (lane == 0)
#pragma unroll
                for (int h = 0; h < 16; ++h) redm[warp * 16 + h] = mx[h];
            named_bar_sync(1, 128);
#pragma unroll
            for (int h = 0; h < 16; ++h)
                mx[h] = fmaxf(fmaxf(redm[h], redm[16 + h]), fmaxf(redm[32 + h], redm[48 + h]));
            float ls[16];
#pragma unroll
            for (int h = 0; h < 16; ++h) ls[h] = 0.f;
            for (int pp = 0; pp < npairs; ++pp) {
                uint32_t r[16];
                tmem_ld16(lanebase + sb * 128 + pp * 16, r);
                tmem_wait_ld16(r);
                const int un = 2 * pp + unit_off;
                const bool valid = un < nu && (un < 16 ? (u[un] * 64 + tok_off <= t) : false);
                const int key = pp * 128 + kl;
                const uint32_t cbase = sP + (key >> 6) * 2048;
                const int kk = key & 63;
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    float e = 0.f;
                    if (valid && mx[h] != -INFINITY) e = exp2f(__uint_as_float(r[h]) * p.scale_log2 - mx[h]);
                    ls[h] += e;
                    __nv_bfloat16 eb = __float2bfloat16_rn(e);
                    st_shared_u16(cbase + sw128_off(h, kk >> 3) + (kk & 7) * 2,
                                  *reinterpret_cast<uint16_t*>(&eb));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sfree[sb]);
            fence_proxy_async_smem();
            mbar_arrive(pfull);
#pragma unroll
            for (int h = 0; h < 16; ++h) {
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) ls[h] += __shfl_xor_sync(0xffffffffu, ls[h], o);
            }
            if (lane == 0)
#pragma unroll
                for (int h = 0; h < 16; ++h) redl[warp * 16 + h] = ls[h];
            named_bar_sync(1, 128);
#pragma unroll
            for (int h = 0; h < 16; ++h) ls[h] = redl[h] + redl[16 + h] + redl[32 + h] + redl[48 + h];

            // O^T: lane = value channel kl, columns = heads
            if (ok) ok = wait_or_abort(&ofull[sb], (i >> 1) & 1, 0x309, abort_flag);
            tc_fence_after();
            uint32_t r[16];
            tmem_ld16(lanebase + 256 + sb * 16, r);
            tmem_wait_ld16(r);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ofree[sb]);
            if (ok && kl < DV) {
                for (int h = 0; h < HG; ++h) {
                    const size_t rowid = ((size_t)b * p.T + t) * p.H + g * HG + h;
                    const float gate = p.gates[rowid * 3 + 1];
                    const float o = ls[h] > 0.f ? __uint_as_float(r[h]) / ls[h] : 0.f;
                    p.out[rowid * DV + kl] += gate * o;
                }
            }
            if (ok && kl < HG && p.lse_user) {
                const size_t rowid = ((size_t)b * p.T + t) * p.H + g * HG + kl;
                p.lse_user[rowid * 3 + 1] = ls[kl] > 0.f ? (mx[kl] + log2f(ls[kl])) * kLn2 : -INFINITY;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace nsa
