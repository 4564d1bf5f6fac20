// k_bwd_kv.cuh -- key-centric backward of the three NSA branches on tcgen05
// tensor cores (pages: natively trainable design; 效率分析 training speed).
//
// With the selection held fixed, the key/value gradients of one branch are,
// for every key u it reads (P = exp(S - LSE), dO_c = g_c dO, D_c = <dO_c, o_c>):
//   dV_u = sum over query rows r that see u of P[r,u] g_r dO_r
//   dK_u = scale * sum over those rows of dS[r,u] q_r,   dS = P (g dP - D),
//   dP[r,u] = <dO_r, v_u>.
// One CTA owns a tile of 128 keys of one (batch, GQA group) -- 128 consecutive
// tokens for the window, 128 compressed blocks for the compressed branch, a
// pair of selection blocks (2m, 2m+1) for the selected branch -- and walks the
// query rows that read them in steps of 64 rows (64/HG tokens x HG heads):
//   S^T  = K Q^T       M = 128 keys, N = 64 rows, K = d_k   (TMEM)
//   dP^T = V dO^T      M = 128 keys, N = 64 rows, K = d_v   (TMEM)
//   softmax warps (thread = key): gP^T = g P^T and dS^T back to TMEM (bf16)
//   dV  += gP^T dO     M = 128 keys, N = d_v, K = 64 rows   (TMEM accumulator)
//   dK  += dS^T Q      M = 128 keys, N = d_k, K = 64 rows   (TMEM accumulator)
// The last two read gP^T / dS^T from tensor memory and take Q / dO as
// transposed (MN-major) operands straight from the tiles the first two read
// K-major, so each row tile is staged once (three stages in flight).  The
// accumulated tile is added into dk/dv (dK~/dV~ for the compressed branch) in
// fp32 at the end; several CTAs can share a key tile (token chunks).
//
// Rows come from consecutive tokens (window, compressed: TMA boxes of 64/HG
// tokens x HG heads) or, for the selected branch, from the tokens that chose
// block 2m or 2m+1 (a list built from the selection; 16-byte copies gather
// their rows).  A row's statistics (log2-domain LSE, D = g <dO, o>, g) come
// from the per-query pass of the backward.
//
// Warps 0-7: softmax and epilogue (a key per TMEM lane, warps 4-7 taking the
// second half of each step's rows); warp 8: loader (TMA, or gather with warp
// 10); warp 9: MMA issuer and TMEM owner.
#pragma once
#include "nsa_dev.cuh"
#include "k_attn_packed.cuh"
#include "k_backward.cuh"

namespace nsa {

constexpr int kBkvRows = 64;        // query rows per step
constexpr int kBkvChunk = 256;      // tokens (or list entries) per CTA

// Shared-memory descriptor of an MN-major operand tile in the 128-byte swizzle
// layout: rows along K of 128 bytes (64 bf16 of the M/N dimension), 8-row atoms
// of 1024 bytes; further 64-element column blocks of M/N `lbo` bytes apart,
// further 8-row groups along K `sbo` bytes apart.
__device__ __forceinline__ uint64_t sdesc_sw128_mn(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// kind::f16 instruction descriptor with the B operand MN-major (transposed)
__host__ __device__ constexpr uint32_t idesc_bf16_bmn(int M, int N) { return idesc_bf16(M, N) | (1u << 16); }

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

__device__ __forceinline__ void red_add_v1(float* p, float a) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(a) : "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

template <int DK, int DV>
struct BkvCfg {
    static constexpr int NQB = DK / 64, NVB = DV / 64;
    static constexpr int NST = 3;                      // stages of query rows in flight
    static constexpr int kKTile = 128 * DK * 2;        // NQB boxes [128 keys][64]
    static constexpr int kVTile = 128 * DV * 2;
    static constexpr int kQStage = kBkvRows * DK * 2;  // NQB boxes [64 rows][64]
    static constexpr int kOStage = kBkvRows * DV * 2;
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + kKTile;
    static constexpr int kOffQ = kOffV + kVTile;
    static constexpr int kOffO = kOffQ + NST * kQStage;
    static constexpr int kOffStat = kOffO + NST * kOStage;   // NST stages x 5 arrays x 64
    static constexpr int kStatBytes = 5 * kBkvRows * 4;
    static constexpr int kOffBar = kOffStat + NST * kStatBytes;
    static constexpr int kSmem = kOffBar + 256 + 1024;
    static_assert(kSmem <= 232448, "shared memory");
    static constexpr int kThreads = 352;
    // TMEM columns: S^T 0, gP^T 64 and dS^T 96 (bf16 pairs: the A operands of the
    // gradient products), dP^T 128, dV 192, dK 192 + DV
    static constexpr uint32_t kColGP = 64, kColDS = 96, kColDP = 128, kColDV = 192, kColDK = 192 + DV;
    static_assert(kColDK + DK <= 512, "tensor memory");
};

struct BkvParams {
    BwdParams bp;
    int n_pairs;            // selection block pairs per (b, g)
    const int* poff;        // [B*G*n_pairs + 1] list offsets
    const int* pcnt;        // [B*G*n_pairs]
    const int* pchunk;      // [B*G*n_pairs + 1] chunk prefix
    const int* plist;       // entries t | (halves << 30)
};

template <int DK, int DV, int HG, int BR>
__global__ void __launch_bounds__(352, 1)
    bwd_kv_tc(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
              const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapO,
              const BkvParams P) {
    using Cfg = BkvCfg<DK, DV>;
    constexpr int TPS = kBkvRows / HG;              // tokens per step
    const BwdParams& p = P.bp;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));

    // ---------------------------------------------------------- work item
    int b, g, key0, tok_lo, tok_hi;
    if (BR == kBrSlc) {
        const int total = P.pchunk[p.B * p.G * P.n_pairs];
        const int cid = blockIdx.x;
        if (cid >= total) return;
        int lo = 0, hi = p.B * p.G * P.n_pairs;     // pair entry e with pchunk[e] <= cid < pchunk[e+1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (P.pchunk[mid] <= cid) lo = mid;
            else hi = mid;
        }
        const int e = lo;
        b = e / (p.G * P.n_pairs);
        g = (e / P.n_pairs) % p.G;
        key0 = (e % P.n_pairs) * 128;
        tok_lo = P.poff[e] + (cid - P.pchunk[e]) * kBkvChunk;
        tok_hi = min(P.poff[e] + P.pcnt[e], tok_lo + kBkvChunk);
    } else {
        b = blockIdx.z / p.G;
        g = blockIdx.z % p.G;
        key0 = blockIdx.x * 128;
        if (BR == kBrWin) {
            if (key0 >= p.T) return;
            const int tmax = min(p.T, key0 + 128 + p.w - 1);
            tok_lo = key0 + blockIdx.y * kBkvChunk;
            tok_hi = min(tmax, tok_lo + kBkvChunk);
        } else {
            if (key0 >= p.C) return;
            tok_lo = key0 * p.d + p.l - 1 + blockIdx.y * kBkvChunk;
            tok_hi = min(p.T, tok_lo + kBkvChunk);
        }
    }
    if (tok_lo >= tok_hi) return;
    const int nsteps = (tok_hi - tok_lo + TPS - 1) / TPS;
    const int nkeys = BR == kBrCmp ? p.C : p.T;

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
    uint64_t* kvfull = bars + 0;
    uint64_t* stfull = bars + 1;    // [NST]
    uint64_t* stempty = bars + 4;   // [NST]
    uint64_t* sfull = bars + 7;
    uint64_t* sfree = bars + 8;
    uint64_t* dpfull = bars + 9;
    uint64_t* dpfree = bars + 10;
    uint64_t* pfull = bars + 11;
    uint64_t* pempty = bars + 12;
    uint64_t* accfull = bars + 13;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 15);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        mbar_init(kvfull, 1);
        for (int s = 0; s < Cfg::NST; ++s) {
            mbar_init(&stfull[s], BR == kBrSlc ? 2 : 1);
            mbar_init(&stempty[s], 1);
        }
        mbar_init(sfull, 1);
        mbar_init(sfree, 8);
        mbar_init(dpfull, 1);
        mbar_init(dpfree, 8);
        mbar_init(pfull, 8);
        mbar_init(pempty, 1);
        mbar_init(accfull, 1);
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

    float* st_lse = reinterpret_cast<float*>(smem + Cfg::kOffStat);      // [NST][5][64]
    auto stat = [&](int st, int a) -> float* { return st_lse + (st * 5 + a) * kBkvRows; };
    // warp-collective wait: lane 0 polls, every lane gets the outcome
    auto lane0_wait = [&](uint64_t* bar, uint32_t parity, unsigned site) -> bool {
        bool ok = true;
        if (lane == 0) ok = wait_or_abort(bar, parity, site, abort_flag);
        return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    };

    if (warp == 8 || (BR == kBrSlc && warp == 10)) {
        // -------------------------------------------------------- loader
        if (warp == 8) {                            // the key tile (rows past the keys: zeros)
            if (lane == 0) mbar_expect_tx(kvfull, Cfg::kKTile + Cfg::kVTile);
            __syncwarp();
            if (lane < Cfg::NQB)
                tma_load_4d(smem + Cfg::kOffK + lane * 16384, &mapK, kvfull, lane * 64, g, key0, b);
            else if (lane < Cfg::NQB + Cfg::NVB)
                tma_load_4d(smem + Cfg::kOffV + (lane - Cfg::NQB) * 16384, &mapV, kvfull,
                            (lane - Cfg::NQB) * 64, g, key0, b);
        }
        if (BR != kBrSlc) {
            // a step's row statistics are read into registers one step ahead, so
            // their latency overlaps the previous step
            float rl[2], rd[2], rg[2];
            int rt[2];
            auto load_stats = [&](int j) {
                const int t0 = tok_lo + j * TPS;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int cc = lane + 32 * half;
                    const int t = t0 + cc / HG, h = cc % HG;
                    const bool valid = t < tok_hi;
                    const size_t r3 = (((size_t)b * p.T + (valid ? t : 0)) * p.H + (size_t)g * HG + h) * 3 + BR;
                    rl[half] = valid ? p.lse2[r3] : INFINITY;
                    rd[half] = valid ? p.dlt[r3] : 0.f;
                    rg[half] = valid ? p.gates[r3] : 0.f;
                    rt[half] = valid ? t : -1;
                }
            };
            load_stats(0);
            for (int j = 0; j < nsteps; ++j) {
                const int st = j % Cfg::NST;
                const int t0 = tok_lo + j * TPS;
                if (j >= Cfg::NST && !lane0_wait(&stempty[st], ((j / Cfg::NST) - 1) & 1, 0x401)) break;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int cc = lane + 32 * half;
                    stat(st, 0)[cc] = rl[half];
                    stat(st, 1)[cc] = rd[half];
                    stat(st, 2)[cc] = rg[half];
                    reinterpret_cast<int*>(stat(st, 3))[cc] = rt[half];
                    reinterpret_cast<int*>(stat(st, 4))[cc] = 3;
                }
                __syncwarp();
                if (lane == 0) mbar_expect_tx(&stfull[st], Cfg::kQStage + Cfg::kOStage);
                __syncwarp();
                if (lane < Cfg::NQB)
                    tma_load_4d(smem + Cfg::kOffQ + st * Cfg::kQStage + lane * 8192, &mapQ, &stfull[st],
                                lane * 64, g * HG, t0, b);
                else if (lane < Cfg::NQB + Cfg::NVB)
                    tma_load_4d(smem + Cfg::kOffO + st * Cfg::kOStage + (lane - Cfg::NQB) * 8192, &mapO,
                                &stfull[st], (lane - Cfg::NQB) * 64, g * HG, t0, b);
                if (j + 1 < nsteps) load_stats(j + 1);
            }
        } else {
            // gather: thread cc (0..63) stages query row cc of each step with 16-byte
            // copies into the 128-byte-swizzled tiles.  A step is posted as soon as its
            // copies land, before the wait for the next stage: the MMA that frees that
            // stage runs only after the posted step's products have been issued.  The
            // list entry and row statistics of a step are read one step ahead.
            const int cc = (warp == 8 ? 0 : 32) + lane;
            const int tk = cc / HG, h = cc % HG;
            bool valid;
            int ent;
            float rl, rd, rg;
            auto load_entry = [&](int j) {
                const int e = tok_lo + j * TPS + tk;
                valid = e < tok_hi;
                ent = valid ? __ldg(P.plist + e) : 0;
                const size_t row = ((size_t)b * p.T + (ent & 0x3FFFFFFF)) * p.H + (size_t)g * HG + h;
                rl = valid ? p.lse2[row * 3 + BR] : INFINITY;
                rd = valid ? p.dlt[row * 3 + BR] : 0.f;
                rg = valid ? p.gates[row * 3 + BR] : 0.f;
            };
            load_entry(0);
            for (int j = 0; j <= nsteps; ++j) {
                if (j >= 1) {
                    asm volatile("cp.async.wait_group 0;" ::: "memory");
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&stfull[(j - 1) % Cfg::NST]);
                }
                if (j == nsteps) break;
                const int st = j % Cfg::NST;
                if (j >= Cfg::NST && !lane0_wait(&stempty[st], ((j / Cfg::NST) - 1) & 1, 0x402)) break;
                const int t = ent & 0x3FFFFFFF;
                const size_t row = ((size_t)b * p.T + t) * p.H + (size_t)g * HG + h;
                stat(st, 0)[cc] = rl;
                stat(st, 1)[cc] = rd;
                stat(st, 2)[cc] = rg;
                reinterpret_cast<int*>(stat(st, 3))[cc] = valid ? t : -1;
                reinterpret_cast<int*>(stat(st, 4))[cc] = (int)((unsigned)ent >> 30);
                const uint32_t sq = smem_u32(smem + Cfg::kOffQ + st * Cfg::kQStage);
                const uint32_t so = smem_u32(smem + Cfg::kOffO + st * Cfg::kOStage);
                if (valid) {
                    const __nv_bfloat16* qr = p.q + row * DK;
                    const __nv_bfloat16* orow = p.dout + row * DV;
#pragma unroll
                    for (int bx = 0; bx < Cfg::NQB; ++bx)
#pragma unroll
                        for (int c = 0; c < 8; ++c) cp_async16(sq + bx * 8192 + sw128_off(cc, c), qr + bx * 64 + c * 8);
#pragma unroll
                    for (int bx = 0; bx < Cfg::NVB; ++bx)
#pragma unroll
                        for (int c = 0; c < 8; ++c) cp_async16(so + bx * 8192 + sw128_off(cc, c), orow + bx * 64 + c * 8);
                } else {                            // rows past the list: zeros (finite operands)
#pragma unroll
                    for (int bx = 0; bx < Cfg::NQB; ++bx)
#pragma unroll
                        for (int c = 0; c < 8; ++c) st_shared_v4(sq + bx * 8192 + sw128_off(cc, c), 0, 0, 0, 0);
#pragma unroll
                    for (int bx = 0; bx < Cfg::NVB; ++bx)
#pragma unroll
                        for (int c = 0; c < 8; ++c) st_shared_v4(so + bx * 8192 + sw128_off(cc, c), 0, 0, 0, 0);
                }
                asm volatile("cp.async.commit_group;" ::: "memory");
                if (j + 1 < nsteps) load_entry(j + 1);
            }
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
    } else if (warp == 9) {
        // ----------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, kBkvRows);
            constexpr uint32_t idV = idesc_bf16_bmn(128, DV);
            constexpr uint32_t idK = idesc_bf16_bmn(128, DK);
            const uint32_t sK = smem_u32(smem + Cfg::kOffK), sV = smem_u32(smem + Cfg::kOffV);
            bool ok = wait_or_abort(kvfull, 0, 0x403, abort_flag);
            // Two independent streams of products: S^T/dP^T of step js (when its rows
            // are staged and its TMEM buffers free) and dV/dK of step jg (when its
            // gP^T/dS^T are written).  Each is issued as soon as it is ready, so the
            // gradient products of a step never wait for the next step's rows.
            int js = 0, jg = 0;
            unsigned long long t_idle = 0;
            uint32_t spins = 0;
            while (ok && jg < nsteps) {
                bool progressed = false;
                if (js < nsteps) {
                    const int st = js % Cfg::NST;
                    const bool ready = mbar_test_wait(&stfull[st], (js / Cfg::NST) & 1) &&
                                       (js < 1 || (mbar_test_wait(sfree, (js - 1) & 1) &&
                                                   mbar_test_wait(dpfree, (js - 1) & 1)));
                    if (ready) {
                        tc_fence_after();
                        const uint32_t sQ = smem_u32(smem + Cfg::kOffQ + st * Cfg::kQStage);
                        const uint32_t sO = smem_u32(smem + Cfg::kOffO + st * Cfg::kOStage);
#pragma unroll
                        for (int kk = 0; kk < DK / 16; ++kk)
                            umma_bf16_ss(tmem, sdesc_sw128(sK + (kk / 4) * 16384 + (kk % 4) * 32),
                                         sdesc_sw128(sQ + (kk / 4) * 8192 + (kk % 4) * 32), idS, kk > 0 ? 1u : 0u);
                        umma_commit(sfull);
#pragma unroll
                        for (int kk = 0; kk < DV / 16; ++kk)
                            umma_bf16_ss(tmem + Cfg::kColDP, sdesc_sw128(sV + (kk / 4) * 16384 + (kk % 4) * 32),
                                         sdesc_sw128(sO + (kk / 4) * 8192 + (kk % 4) * 32), idS, kk > 0 ? 1u : 0u);
                        umma_commit(dpfull);
                        ++js;
                        progressed = true;
                    }
                }
                if (jg < js && mbar_test_wait(pfull, jg & 1)) {
                    const int st = jg % Cfg::NST;
                    tc_fence_after();
                    const uint32_t sQ = smem_u32(smem + Cfg::kOffQ + st * Cfg::kQStage);
                    const uint32_t sO = smem_u32(smem + Cfg::kOffO + st * Cfg::kOStage);
#pragma unroll
                    for (int kk = 0; kk < kBkvRows / 16; ++kk)
                        umma_bf16_ts(tmem + Cfg::kColDV, tmem + Cfg::kColGP + kk * 8,
                                     sdesc_sw128_mn(sO + kk * 2048, 8192, 1024), idV, (jg > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < kBkvRows / 16; ++kk)
                        umma_bf16_ts(tmem + Cfg::kColDK, tmem + Cfg::kColDS + kk * 8,
                                     sdesc_sw128_mn(sQ + kk * 2048, 8192, 1024), idK, (jg > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&stempty[st]);
                    umma_commit(pempty);
                    ++jg;
                    progressed = true;
                }
                // bounded: no progress for the wait limit ends the CTA with an error
                if (progressed) {
                    spins = 0;
                } else if ((++spins & 63u) == 0u) {
                    if (*abort_flag) {
                        ok = false;
                    } else {
                        const unsigned long long now = globaltimer_ns();
                        if (t_idle == 0) t_idle = now;
                        else if (now - t_idle > kWaitLimitNs) {
                            record_timeout(0x404);
                            *abort_flag = 1;
                            ok = false;
                        }
                    }
                }
                if (progressed) t_idle = 0;
            }
            umma_commit(accfull);               // also on the abort path: the epilogue waits on it
        }
    } else if (warp < 8) {
        // ------------------------------------------------- softmax, epilogue
        // warp w: keys 32 (w % 4) .. +31 (its TMEM lane quadrant), query rows
        // 32 (w / 4) .. +31 of each step
        const int quad = warp & 3, hc = warp >> 2;
        const int kl = quad * 32 + lane;                     // key within the tile = TMEM lane
        const int u = key0 + kl;
        const bool key_ok = u < nkeys;
        const int half = kl >> 6;                            // selected branch: block 2m or 2m+1
        const uint32_t lanebase = tmem + ((uint32_t)(quad * 32) << 16);
        const float c = p.scale_log2;
        constexpr int TPH = 32 / HG > 0 ? 32 / HG : 1;       // tokens among this warp's 32 rows
        bool ok = true;
        for (int j = 0; j < nsteps; ++j) {
            const int st = j % Cfg::NST;
            // the step's row statistics (written by the loader before it posted the stage)
            if (!(ok = lane0_wait(&stfull[st], (j / Cfg::NST) & 1, 0x40C))) break;
            if (!(ok = lane0_wait(sfull, j & 1, 0x408))) break;
            if (!(ok = lane0_wait(dpfull, j & 1, 0x409))) break;
            tc_fence_after();
            uint32_t sr[32], dr[32];
            tmem_ld32(lanebase + hc * 32, sr);
            tmem_ld32(lanebase + Cfg::kColDP + hc * 32, dr);
            const float4* L4 = reinterpret_cast<const float4*>(stat(st, 0) + hc * 32);
            const float4* D4 = reinterpret_cast<const float4*>(stat(st, 1) + hc * 32);
            const float4* G4 = reinterpret_cast<const float4*>(stat(st, 2) + hc * 32);
            const int* TK = reinterpret_cast<const int*>(stat(st, 3)) + hc * 32;
            const int* BT = reinterpret_cast<const int*>(stat(st, 4)) + hc * 32;
            // does each of this warp's tokens see this key?
            bool vt[TPH];
#pragma unroll
            for (int tk = 0; tk < TPH; ++tk) {
                const int t = TK[tk * HG];
                bool v = key_ok && t >= 0;
                if constexpr (BR == kBrWin) v = v && u <= t && u > t - p.w;
                else if constexpr (BR == kBrCmp) v = v && u * p.d + p.l - 1 <= t;
                else v = v && u <= t && ((BT[tk * HG] >> half) & 1);
                vt[tk] = v;
            }
            tmem_wait_ld32(sr);
            tmem_wait_ld32(dr);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {                                 // this warp's columns are read
                mbar_arrive(sfree);
                mbar_arrive(dpfree);
            }
            uint32_t gp[16], dsv[16];
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {                 // 4 rows per statistics load
                const float4 l4 = L4[q4], d4 = D4[q4], g4 = G4[q4];
                const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
                const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
                const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
                float pv[4], dsn[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int col = q4 * 4 + e;
                    const float pr = vt[col / HG] ? ex2a(fmaf(__uint_as_float(sr[col]), c, -lv[e])) : 0.f;
                    pv[e] = gv[e] * pr;
                    dsn[e] = pr * fmaf(gv[e], __uint_as_float(dr[col]), -dv[e]);
                }
                gp[q4 * 2] = pack_bf16x2(pv[0], pv[1]);
                gp[q4 * 2 + 1] = pack_bf16x2(pv[2], pv[3]);
                dsv[q4 * 2] = pack_bf16x2(dsn[0], dsn[1]);
                dsv[q4 * 2 + 1] = pack_bf16x2(dsn[2], dsn[3]);
            }
            // the previous step's dV / dK products have read gP^T / dS^T
            if (j >= 1 && !(ok = lane0_wait(pempty, (j - 1) & 1, 0x40A))) break;
            tc_fence_after();
            // this warp's 32 rows: K-steps 2 hc and 2 hc + 1 of the gradient products
            tmem_st16(lanebase + Cfg::kColGP + hc * 16, gp);
            tmem_st16(lanebase + Cfg::kColDS + hc * 16, dsv);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(pfull);
        }
        // epilogue: the tile's dV (warps 0-3) and scale * dK (warps 4-7) added into
        // the fp32 gradients
        if (lane0_wait(accfull, 0, 0x40B) && ok) {
            tc_fence_after();
            const size_t rowk = ((size_t)b * nkeys + (key_ok ? u : 0)) * p.G + g;
            const int ncol = hc == 0 ? DV : DK;
            const uint32_t col0 = hc == 0 ? Cfg::kColDV : Cfg::kColDK;
            float* dst = (hc == 0 ? (BR == kBrCmp ? p.dvc : p.dv) : (BR == kBrCmp ? p.dkc : p.dk)) + rowk * ncol;
            const float sc = hc == 0 ? 1.f : p.scale;
#pragma unroll 1
            for (int c0 = 0; c0 < ncol; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(lanebase + col0 + c0, r);
                tmem_wait_ld32(r);
                if (key_ok) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        red_add_v4(dst + c0 + e, sc * __uint_as_float(r[e]), sc * __uint_as_float(r[e + 1]),
                                   sc * __uint_as_float(r[e + 2]), sc * __uint_as_float(r[e + 3]));
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

// ------------------------------------ selected branch: block pairs -> tokens
// For every (b, t, g) row of the selection, each distinct pair m = j/2 of its
// selected blocks j, with bit h set when block 2m + h was chosen: emit(m, bits)
// once per pair (the row is ascending, so a pair's blocks are adjacent).
template <typename F>
__device__ __forceinline__ void for_each_pair(const int32_t* r, int n, int nsb, F&& emit) {
    int cur = -1, bits = 0;
    for (int a = 0; a < n; ++a) {
        const int j = r[a];
        if (j < 0 || j >= nsb) break;
        const int m = j >> 1;
        if (m != cur) {
            if (cur >= 0) emit(cur, bits);
            cur = m;
            bits = 0;
        }
        bits |= 1 << (j & 1);
    }
    if (cur >= 0) emit(cur, bits);
}

__global__ void bwd_pair_count(const BwdParams p, int n_pairs, int* pcnt) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)p.B * p.T * p.G) return;
    const int g = (int)(i % p.G);
    const int b = (int)(i / ((long long)p.T * p.G));
    int* base = pcnt + ((size_t)b * p.G + g) * n_pairs;
    for_each_pair(p.idx + i * p.n, p.n, p.NSb, [&](int m, int) { atomicAdd(base + m, 1); });
}

// single CTA: poff = exclusive scan of pcnt, pchunk = scan of ceil(pcnt / chunk)
__global__ void __launch_bounds__(1024) bwd_pair_scan(int N, const int* pcnt, int* poff, int* pchunk) {
    __shared__ int s_cnt[1024], s_ch[1024];
    const int per = (N + 1023) / 1024;
    const int beg = min(N, (int)threadIdx.x * per), end = min(N, beg + per);
    int a = 0, c = 0;
    for (int i = beg; i < end; ++i) {
        a += pcnt[i];
        c += (pcnt[i] + kBkvChunk - 1) / kBkvChunk;
    }
    s_cnt[threadIdx.x] = a;
    s_ch[threadIdx.x] = c;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
        const int va = threadIdx.x >= (unsigned)o ? s_cnt[threadIdx.x - o] : 0;
        const int vc = threadIdx.x >= (unsigned)o ? s_ch[threadIdx.x - o] : 0;
        __syncthreads();
        s_cnt[threadIdx.x] += va;
        s_ch[threadIdx.x] += vc;
        __syncthreads();
    }
    a = s_cnt[threadIdx.x] - a;
    c = s_ch[threadIdx.x] - c;
    for (int i = beg; i < end; ++i) {
        poff[i] = a;
        pchunk[i] = c;
        a += pcnt[i];
        c += (pcnt[i] + kBkvChunk - 1) / kBkvChunk;
    }
    if (threadIdx.x == 1023) {
        poff[N] = s_cnt[1023];
        pchunk[N] = s_ch[1023];
    }
}

__global__ void bwd_pair_fill(const BwdParams p, int n_pairs, const int* poff, int* cursor, int* plist) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)p.B * p.T * p.G) return;
    const int g = (int)(i % p.G);
    const int t = (int)((i / p.G) % p.T);
    const int b = (int)(i / ((long long)p.T * p.G));
    const size_t e0 = ((size_t)b * p.G + g) * n_pairs;
    for_each_pair(p.idx + i * p.n, p.n, p.NSb, [&](int m, int bits) {
        const int pos = atomicAdd(&cursor[e0 + m], 1);
        plist[poff[e0 + m] + pos] = (int)((unsigned)t | ((unsigned)bits << 30));
    });
}

}  // namespace nsa
