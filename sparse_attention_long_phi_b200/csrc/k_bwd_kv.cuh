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
//   S^T  = K Q^T       M = 128 keys, N = 64 rows, K = d_k   (TMEM, 2 buffers)
//   dP^T = V dO^T      M = 128 keys, N = 64 rows, K = d_v   (TMEM)
//   softmax warps (thread = key): gP^T = g P^T and dS^T to shared memory (bf16)
//   dV  += gP^T dO     M = 128 keys, N = d_v, K = 64 rows   (TMEM accumulator)
//   dK  += dS^T Q      M = 128 keys, N = d_k, K = 64 rows   (TMEM accumulator)
// The last two take Q / dO as transposed (MN-major) operands straight from the
// tiles the first two read K-major, so each row tile is staged once.  The
// accumulated tile is added into dk/dv (dK~/dV~ for the compressed branch) in
// fp32 at the end; several CTAs can share a key tile (token chunks).
//
// Rows come from consecutive tokens (window, compressed: TMA boxes of 64/HG
// tokens x HG heads) or, for the selected branch, from the tokens that chose
// block 2m or 2m+1 (a list built from the selection; 16-byte copies gather
// their rows).  A row's statistics (log2-domain LSE, D = g <dO, o>, g) come
// from the per-query pass of the backward.
//
// Warps 0-3: softmax and epilogue (thread = key = TMEM lane); warp 4: loader
// (TMA, or gather with warp 6); warp 5: MMA issuer and TMEM owner.
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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

template <int DK, int DV>
struct BkvCfg {
    static constexpr int NQB = DK / 64, NVB = DV / 64;
    static constexpr int kKTile = 128 * DK * 2;        // NQB boxes [128 keys][64]
    static constexpr int kVTile = 128 * DV * 2;
    static constexpr int kQStage = kBkvRows * DK * 2;  // NQB boxes [64 rows][64]
    static constexpr int kOStage = kBkvRows * DV * 2;
    static constexpr int kPT = 128 * kBkvRows * 2;     // gP^T / dS^T: [128 keys][64 rows]
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + kKTile;
    static constexpr int kOffQ = kOffV + kVTile;
    static constexpr int kOffO = kOffQ + 2 * kQStage;
    static constexpr int kOffGP = kOffO + 2 * kOStage;
    static constexpr int kOffDS = kOffGP + kPT;
    static constexpr int kOffStat = kOffDS + kPT;      // 2 stages x 5 arrays x 64
    static constexpr int kStatBytes = 5 * kBkvRows * 4;
    static constexpr int kOffBar = kOffStat + 2 * kStatBytes;
    static constexpr int kSmem = kOffBar + 256 + 1024;
    static_assert(kSmem <= 232448, "shared memory");
    static constexpr int kThreads = 224;
    // TMEM columns: S^T buffers 0 / 64, dP^T 128, dV 192, dK 192 + DV
    static constexpr uint32_t kColDP = 128, kColDV = 192, kColDK = 192 + DV;
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
__global__ void __launch_bounds__(224, 1)
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
    uint64_t* stfull = bars + 1;    // [2]
    uint64_t* stempty = bars + 3;   // [2]
    uint64_t* sfull = bars + 5;     // [2]
    uint64_t* sfree = bars + 7;     // [2]
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
        for (int s = 0; s < 2; ++s) {
            mbar_init(&stfull[s], BR == kBrSlc ? 2 : 1);
            mbar_init(&stempty[s], 1);
            mbar_init(&sfull[s], 1);
            mbar_init(&sfree[s], 4);
        }
        mbar_init(dpfull, 1);
        mbar_init(dpfree, 4);
        mbar_init(pfull, 4);
        mbar_init(pempty, 1);
        mbar_init(accfull, 1);
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

    float* st_lse = reinterpret_cast<float*>(smem + Cfg::kOffStat);      // [2][5][64]
    auto stat = [&](int st, int a) -> float* { return st_lse + (st * 5 + a) * kBkvRows; };
    // warp-collective wait: lane 0 polls, every lane gets the outcome
    auto lane0_wait = [&](uint64_t* bar, uint32_t parity, unsigned site) -> bool {
        bool ok = true;
        if (lane == 0) ok = wait_or_abort(bar, parity, site, abort_flag);
        return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    };

    if (warp == 4 || (BR == kBrSlc && warp == 6)) {
        // -------------------------------------------------------- loader
        if (warp == 4) {                            // the key tile (rows past the keys: zeros)
            if (lane == 0) mbar_expect_tx(kvfull, Cfg::kKTile + Cfg::kVTile);
            __syncwarp();
            if (lane < Cfg::NQB)
                tma_load_4d(smem + Cfg::kOffK + lane * 16384, &mapK, kvfull, lane * 64, g, key0, b);
            else if (lane < Cfg::NQB + Cfg::NVB)
                tma_load_4d(smem + Cfg::kOffV + (lane - Cfg::NQB) * 16384, &mapV, kvfull,
                            (lane - Cfg::NQB) * 64, g, key0, b);
        }
        if (BR != kBrSlc) {
            for (int j = 0; j < nsteps; ++j) {
                const int st = j & 1;
                if (j >= 2 && !lane0_wait(&stempty[st], ((j - 2) >> 1) & 1, 0x401)) break;
                const int t0 = tok_lo + j * TPS;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int cc = lane + 32 * half;
                    const int t = t0 + cc / HG, h = cc % HG;
                    const bool valid = t < tok_hi;
                    const size_t r3 = (((size_t)b * p.T + (valid ? t : 0)) * p.H + (size_t)g * HG + h) * 3 + BR;
                    stat(st, 0)[cc] = valid ? p.lse2[r3] : INFINITY;
                    stat(st, 1)[cc] = valid ? p.dlt[r3] : 0.f;
                    stat(st, 2)[cc] = valid ? p.gates[r3] : 0.f;
                    reinterpret_cast<int*>(stat(st, 3))[cc] = valid ? t : -1;
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
            }
        } else {
            // gather: thread cc (0..63) stages query row cc of each step with 16-byte
            // copies into the 128-byte-swizzled tiles.  A step is posted as soon as its
            // copies land, before the wait for the next stage: the MMA that frees that
            // stage runs only after the posted step's products have been issued.
            const int cc = (warp == 4 ? 0 : 32) + lane;
            const int tk = cc / HG, h = cc % HG;
            for (int j = 0; j <= nsteps; ++j) {
                if (j >= 1) {
                    asm volatile("cp.async.wait_group 0;" ::: "memory");
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&stfull[(j - 1) & 1]);
                }
                if (j == nsteps) break;
                const int st = j & 1;
                if (j >= 2 && !lane0_wait(&stempty[st], ((j - 2) >> 1) & 1, 0x402)) break;
                const int e = tok_lo + j * TPS + tk;
                const bool valid = e < tok_hi;
                const int ent = valid ? P.plist[e] : 0;
                const int t = ent & 0x3FFFFFFF;
                const size_t row = ((size_t)b * p.T + t) * p.H + (size_t)g * HG + h;
                stat(st, 0)[cc] = valid ? p.lse2[row * 3 + BR] : INFINITY;
                stat(st, 1)[cc] = valid ? p.dlt[row * 3 + BR] : 0.f;
                stat(st, 2)[cc] = valid ? p.gates[row * 3 + BR] : 0.f;
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
            }
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
    } else if (warp == 5) {
        // ----------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, kBkvRows);
            constexpr uint32_t idV = idesc_bf16_bmn(128, DV);
            constexpr uint32_t idK = idesc_bf16_bmn(128, DK);
            const uint32_t sK = smem_u32(smem + Cfg::kOffK), sV = smem_u32(smem + Cfg::kOffV);
            const uint32_t sGP = smem_u32(smem + Cfg::kOffGP), sDS = smem_u32(smem + Cfg::kOffDS);
            bool ok = wait_or_abort(kvfull, 0, 0x403, abort_flag);
            auto grad = [&](int i) -> bool {
                const int st = i & 1;
                if (!wait_or_abort(pfull, i & 1, 0x404, abort_flag)) return false;
                tc_fence_after();
                const uint32_t sQ = smem_u32(smem + Cfg::kOffQ + st * Cfg::kQStage);
                const uint32_t sO = smem_u32(smem + Cfg::kOffO + st * Cfg::kOStage);
#pragma unroll
                for (int kk = 0; kk < kBkvRows / 16; ++kk)
                    umma_bf16_ss(tmem + Cfg::kColDV, sdesc_sw128(sGP + kk * 32),
                                 sdesc_sw128_mn(sO + kk * 2048, 8192, 1024), idV, (i > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < kBkvRows / 16; ++kk)
                    umma_bf16_ss(tmem + Cfg::kColDK, sdesc_sw128(sDS + kk * 32),
                                 sdesc_sw128_mn(sQ + kk * 2048, 8192, 1024), idK, (i > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&stempty[st]);
                umma_commit(pempty);
                return true;
            };
            for (int j = 0; j < nsteps && ok; ++j) {
                const int st = j & 1;
                if (!(ok = wait_or_abort(&stfull[st], (j >> 1) & 1, 0x405, abort_flag))) break;
                if (j >= 2 && !(ok = wait_or_abort(&sfree[st], ((j - 2) >> 1) & 1, 0x406, abort_flag))) break;
                tc_fence_after();
                const uint32_t sQ = smem_u32(smem + Cfg::kOffQ + st * Cfg::kQStage);
                const uint32_t sO = smem_u32(smem + Cfg::kOffO + st * Cfg::kOStage);
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)
                    umma_bf16_ss(tmem + st * 64, sdesc_sw128(sK + (kk / 4) * 16384 + (kk % 4) * 32),
                                 sdesc_sw128(sQ + (kk / 4) * 8192 + (kk % 4) * 32), idS, kk > 0 ? 1u : 0u);
                umma_commit(&sfull[st]);
                if (j >= 1 && !(ok = wait_or_abort(dpfree, (j - 1) & 1, 0x407, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < DV / 16; ++kk)
                    umma_bf16_ss(tmem + Cfg::kColDP, sdesc_sw128(sV + (kk / 4) * 16384 + (kk % 4) * 32),
                                 sdesc_sw128(sO + (kk / 4) * 8192 + (kk % 4) * 32), idS, kk > 0 ? 1u : 0u);
                umma_commit(dpfull);
                if (j >= 1) ok = grad(j - 1);
            }
            if (ok) ok = grad(nsteps - 1);
            umma_commit(accfull);               // also on the abort path: the epilogue waits on it
        }
    } else if (warp < 4) {
        // ------------------------------------------------- softmax, epilogue
        const int kl = warp * 32 + lane;                     // key within the tile = TMEM lane
        const int u = key0 + kl;
        const bool key_ok = u < nkeys;
        const int half = kl >> 6;                            // selected branch: block 2m or 2m+1
        const uint32_t lanebase = tmem + ((uint32_t)(warp * 32) << 16);
        const uint32_t rowGP = smem_u32(smem + Cfg::kOffGP), rowDS = smem_u32(smem + Cfg::kOffDS);
        const float c = p.scale_log2;
        bool ok = true;
        for (int j = 0; j < nsteps; ++j) {
            const int st = j & 1;
            // the step's row statistics (written by the loader before it posted the stage)
            if (!(ok = lane0_wait(&stfull[st], (j >> 1) & 1, 0x40C))) break;
            if (!(ok = lane0_wait(&sfull[st], (j >> 1) & 1, 0x408))) break;
            if (!(ok = lane0_wait(dpfull, j & 1, 0x409))) break;
            tc_fence_after();
            const float4* L4 = reinterpret_cast<const float4*>(stat(st, 0));
            const float4* D4 = reinterpret_cast<const float4*>(stat(st, 1));
            const float4* G4 = reinterpret_cast<const float4*>(stat(st, 2));
            const int* TK = reinterpret_cast<const int*>(stat(st, 3));
            const int* BT = reinterpret_cast<const int*>(stat(st, 4));
            // does each of the step's tokens see this key?
            bool vt[TPS];
#pragma unroll
            for (int tk = 0; tk < TPS; ++tk) {
                const int t = TK[tk * HG];
                bool v = key_ok && t >= 0;
                if constexpr (BR == kBrWin) v = v && u <= t && u > t - p.w;
                else if constexpr (BR == kBrCmp) v = v && u * p.d + p.l - 1 <= t;
                else v = v && u <= t && ((BT[tk * HG] >> half) & 1);
                vt[tk] = v;
            }
            // two halves of 32 rows: S^T and dP^T columns, then gP^T and dS^T in bf16
            // pairs, stored as soon as the previous step's dV / dK products have read
            // the tiles
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t sr[32], dr[32];
                tmem_ld32(lanebase + st * 64 + hf * 32, sr);
                tmem_ld32(lanebase + Cfg::kColDP + hf * 32, dr);
                tmem_wait_ld32(sr);
                tmem_wait_ld32(dr);
                if (hf == 1) {                      // both TMEM buffers read: release them
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&sfree[st]);
                        mbar_arrive(dpfree);
                    }
                }
                uint32_t gp[16], dsv[16];
#pragma unroll
                for (int q4 = 0; q4 < 8; ++q4) {    // 4 columns per statistics load
                    const int c0 = hf * 32 + q4 * 4;
                    const float4 l4 = L4[c0 / 4], d4 = D4[c0 / 4], g4 = G4[c0 / 4];
                    const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
                    const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
                    const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
                    float pv[4], dsn[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int col = c0 + e;
                        const float sv = __uint_as_float(sr[q4 * 4 + e]);
                        const float dpv = __uint_as_float(dr[q4 * 4 + e]);
                        const float pr = vt[col / HG] ? ex2a(fmaf(sv, c, -lv[e])) : 0.f;
                        pv[e] = gv[e] * pr;
                        dsn[e] = pr * fmaf(gv[e], dpv, -dv[e]);
                    }
                    gp[q4 * 2] = pack_bf16x2(pv[0], pv[1]);
                    gp[q4 * 2 + 1] = pack_bf16x2(pv[2], pv[3]);
                    dsv[q4 * 2] = pack_bf16x2(dsn[0], dsn[1]);
                    dsv[q4 * 2 + 1] = pack_bf16x2(dsn[2], dsn[3]);
                }
                if (hf == 0 && j >= 1 && !(ok = lane0_wait(pempty, (j - 1) & 1, 0x40A))) break;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    st_shared_v4(rowGP + sw128_off(kl, hf * 4 + ch), gp[4 * ch], gp[4 * ch + 1], gp[4 * ch + 2],
                                 gp[4 * ch + 3]);
                    st_shared_v4(rowDS + sw128_off(kl, hf * 4 + ch), dsv[4 * ch], dsv[4 * ch + 1], dsv[4 * ch + 2],
                                 dsv[4 * ch + 3]);
                }
            }
            if (!ok) break;
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(pfull);
        }
        // epilogue: add the tile's dV and scale * dK into the fp32 gradients
        if (lane0_wait(accfull, 0, 0x40B) && ok) {
            tc_fence_after();
            float* dvb = BR == kBrCmp ? p.dvc : p.dv;
            float* dkb = BR == kBrCmp ? p.dkc : p.dk;
            const size_t rowk = ((size_t)b * nkeys + (key_ok ? u : 0)) * p.G + g;
#pragma unroll 1
            for (int c0 = 0; c0 < DV; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(lanebase + Cfg::kColDV + c0, r);
                tmem_wait_ld32(r);
                if (key_ok) {
                    float* dst = dvb + rowk * DV + c0;
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        red_add_v4(dst + e, __uint_as_float(r[e]), __uint_as_float(r[e + 1]),
                                   __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
                }
            }
#pragma unroll 1
            for (int c0 = 0; c0 < DK; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(lanebase + Cfg::kColDK + c0, r);
                tmem_wait_ld32(r);
                if (key_ok) {
                    float* dst = dkb + rowk * DK + c0;
                    const float sc = p.scale;
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        red_add_v4(dst + e, sc * __uint_as_float(r[e]), sc * __uint_as_float(r[e + 1]),
                                   sc * __uint_as_float(r[e + 2]), sc * __uint_as_float(r[e + 3]));
                }
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

// ------------------------------------ selected branch: block pairs -> tokens
// For every (b, t, g) row of the selection, each distinct pair m = j/2 of its
// selected blocks j, with bit h set when block 2m + h was chosen.
__device__ __forceinline__ int pair_entries(const int32_t* r, int n, int nsb, int (&pr)[16], int (&bits)[16]) {
    int np = 0;
    for (int a = 0; a < n && a < 16; ++a) {
        const int j = r[a];
        if (j < 0 || j >= nsb) break;
        const int m = j >> 1;
        if (np > 0 && pr[np - 1] == m) {
            bits[np - 1] |= 1 << (j & 1);
        } else {
            pr[np] = m;
            bits[np] = 1 << (j & 1);
            ++np;
        }
    }
    return np;
}

__global__ void bwd_pair_count(const BwdParams p, int n_pairs, int* pcnt) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)p.B * p.T * p.G) return;
    const int g = (int)(i % p.G);
    const int b = (int)(i / ((long long)p.T * p.G));
    int pr[16], bits[16];
    const int np = pair_entries(p.idx + i * p.n, p.n, p.NSb, pr, bits);
    for (int a = 0; a < np; ++a) atomicAdd(&pcnt[((size_t)b * p.G + g) * n_pairs + pr[a]], 1);
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
    int pr[16], bits[16];
    const int np = pair_entries(p.idx + i * p.n, p.n, p.NSb, pr, bits);
    for (int a = 0; a < np; ++a) {
        const size_t e = ((size_t)b * p.G + g) * n_pairs + pr[a];
        const int pos = atomicAdd(&cursor[e], 1);
        plist[poff[e] + pos] = (int)((unsigned)t | ((unsigned)bits[a] << 30));
    }
}

}  // namespace nsa
