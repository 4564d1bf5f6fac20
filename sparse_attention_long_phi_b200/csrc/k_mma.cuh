// k_mma.cuh -- warp-level bf16 tensor-core building blocks (mma.sync
// m16n8k16, fp32 accumulate) for the kernels whose M side is the 16 query
// heads of one GQA group at one token: decode and the per-query backward.
// Keys are staged 32 per warp in shared memory with a padded pitch; ldmatrix
// builds the B fragments (non-transposed for Q.K^T-like products, transposed
// for P.V-like ones).
#pragma once
#include "nsa_dev.cuh"

namespace nsa {

// ------------------------------------------------------------ mma helpers
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// copy `rows` rows of `width` bf16 (row stride src_stride elements) into
// shared memory with a padded pitch: 16-byte cp.async chunks, all in flight
// at once; rows >= nvalid are zero-filled.  No commit: the caller groups the
// copies with cp_async_commit and waits with cp_async_wait / cp_async_wait_1.
__device__ __forceinline__ void warp_issue_rows(uint8_t* dst, int pitch, const __nv_bfloat16* src,
                                                size_t src_stride, int rows, int nvalid, int width) {
    const int lane = threadIdx.x & 31;
    const int cpr = width / 8;   // 16-byte chunks per row
    for (int e = lane; e < rows * cpr; e += 32) {
        const int r = e / cpr, c = e % cpr;
        const bool ok = r < nvalid;
        const __nv_bfloat16* sp = ok ? src + (size_t)r * src_stride + c * 8 : src;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst + r * pitch + c * 16)),
                     "l"(sp), "r"(ok ? 16 : 0)
                     : "memory");
    }
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
// all but the most recent group complete
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// 32 rows of W bf16 (W a multiple of 64; row stride `stride` elements) into
// shared memory with pitch W*2+16, rows >= nvalid zero-filled; lane (r0, c0) =
// (lane / 8, lane % 8) copies columns c0, c0+8, ... of rows r0, r0+4, ...,
// so every offset but the row step is a compile-time immediate.  `src` must
// be a valid address even when nvalid <= 0.  No commit.
template <int W>
__device__ __forceinline__ void warp_issue_32rows(uint8_t* dst, const __nv_bfloat16* src, size_t stride, int nvalid) {
    constexpr int PITCH = W * 2 + 16, J = W / 64;
    const int lane = threadIdx.x & 31, c0 = lane & 7, r0 = lane >> 3;
    const uint32_t d = smem_u32(dst) + r0 * PITCH + c0 * 16;
    const __nv_bfloat16* s = src + (size_t)r0 * stride + c0 * 8;
    const size_t step = 4 * stride;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const bool ok = r0 + 4 * k < nvalid;
        const __nv_bfloat16* sk = ok ? s + k * step : src;
        const uint32_t n = ok ? 16u : 0u;
#pragma unroll
        for (int j = 0; j < J; ++j)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d + (4 * k * PITCH + j * 128)),
                         "l"(sk + j * 64), "r"(n)
                         : "memory");
    }
}

// L2 policy for data read once: evicted first, so that small results written
// meanwhile stay cached for the kernels that read them next
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// 32 rows of W bf16 (row stride `stride` elements) into shared memory rows of
// pitch W*2+16 with one bulk (TMA) copy per lane, completing on `bar`, which
// this call arms for the min(nrows, 32) valid rows; the others are zero-filled by
// plain stores.  Bulk copies bypass the L1 miss queue that bounds cp.async
// streaming.  `policy` is an L2 cache policy (see l2_evict_first) for the
// copies.  The caller waits on `bar` (phase parity) and then __syncwarp()s
// before reading.  Earlier generic accesses of the rows are fenced first.
template <int W>
__device__ __forceinline__ void warp_bulk_rows(uint8_t* dst, const __nv_bfloat16* src, size_t stride, int nrows,
                                               uint64_t* bar, uint64_t policy) {
    constexpr int PITCH = W * 2 + 16, BYTES = W * 2;
    const int lane = threadIdx.x & 31;
    nrows = max(0, min(nrows, 32));
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_expect_tx(bar, (uint32_t)(max(nrows, 0) * BYTES));
    __syncwarp();
    uint8_t* row = dst + lane * PITCH;
    if (lane < nrows) {
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
            ::"r"(smem_u32(row)), "l"(src + (size_t)lane * stride), "r"(BYTES), "r"(smem_u32(bar)), "l"(policy)
            : "memory");
    } else {   // rows past the valid ones
#pragma unroll
        for (int c = 0; c < BYTES / 16; ++c) st_shared_v4(smem_u32(row + c * 16), 0u, 0u, 0u, 0u);
    }
}

// issue + commit as one group
__device__ __forceinline__ void warp_copy_rows(uint8_t* dst, int pitch, const __nv_bfloat16* src,
                                               size_t src_stride, int rows, int nvalid, int width) {
    warp_issue_rows(dst, pitch, src, src_stride, rows, nvalid, width);
    cp_async_commit();
}

// the same with a per-row source pointer (nullptr rows are zero-filled)
template <typename RowPtr>
__device__ __forceinline__ void warp_copy_rows_ptr(uint8_t* dst, int pitch, RowPtr rowptr, int rows, int width) {
    const int lane = threadIdx.x & 31;
    const int cpr = width / 8;
    for (int e = lane; e < rows * cpr; e += 32) {
        const int r = e / cpr, c = e % cpr;
        const __nv_bfloat16* src = rowptr(r);
        const bool ok = src != nullptr;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst + r * pitch + c * 16)),
                     "l"(ok ? src + c * 8 : reinterpret_cast<const __nv_bfloat16*>(dst)), "r"(ok ? 16 : 0)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// 16 rows (heads) of D bf16 at `base` (row stride D elements; rows >= nrows
// zero) as A fragments of D/16 k-steps
template <int D>
__device__ __forceinline__ void load_a_frags(const __nv_bfloat16* base, int nrows, uint32_t (&a)[D / 16][4]) {
    const int lane = threadIdx.x & 31, gr = lane >> 2, tg = lane & 3;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int c = kk * 16 + tg * 2;
        auto ld = [&](int row, int col) -> uint32_t {
            return row < nrows ? *reinterpret_cast<const uint32_t*>(base + (size_t)row * D + col) : 0u;
        };
        a[kk][0] = ld(gr, c);
        a[kk][1] = ld(gr + 8, c);
        a[kk][2] = ld(gr, c + 8);
        a[kk][3] = ld(gr + 8, c + 8);
    }
}

// S[16 heads x 32 keys] = Q K^T for the warp's 32 keys staged at `ks` (pitch
// DK*2+16), logits scaled to log2 units; sfr[nt][0..3] in accumulator layout
template <int DK>
__device__ __forceinline__ void warp_logits(const uint32_t (&qa)[DK / 16][4], uint32_t ks, float (&sfr)[4][4]) {
    const int lane = threadIdx.x & 31;
    constexpr int pitch = DK * 2 + 16;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sfr[nt][e] = 0.f;
    // ldmatrix x4 (non-transposed): matrices (keys 8nt..+7, dims 16kk..+7),
    // (same keys, dims +8), then the same for n-tile nt+1
    const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
    for (int kk = 0; kk < DK / 16; ++kk) {
#pragma unroll
        for (int nt = 0; nt < 4; nt += 2) {
            const int key = (nt + (mi >> 1)) * 8 + rr;
            const int dim = kk * 16 + (mi & 1) * 8;
            uint32_t b0, b1, b2, b3;
            ldsm_x4(ks + key * pitch + dim * 2, b0, b1, b2, b3);
            mma16816(sfr[nt], qa[kk], b0, b1);
            mma16816(sfr[nt + 1], qa[kk], b2, b3);
        }
    }
}

// the same product with the A side (16 rows of D bf16, pitch D*2+16) staged
// in shared memory at `as` and read with ldmatrix per k-step
template <int D>
__device__ __forceinline__ void warp_logits_sa(uint32_t as, uint32_t ks, float (&sfr)[4][4]) {
    const int lane = threadIdx.x & 31;
    constexpr int pitch = D * 2 + 16;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sfr[nt][e] = 0.f;
    const int mi = lane >> 3, rr = lane & 7;
    // A matrices: (rows 0-7, k 0-7), (rows 8-15, k 0-7), (rows 0-7, k 8-15), (rows 8-15, k 8-15)
    const uint32_t arow = as + ((mi & 1) * 8 + rr) * pitch + (mi >> 1) * 16;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        ldsm_x4(arow + kk * 32, a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int nt = 0; nt < 4; nt += 2) {
            const int key = (nt + (mi >> 1)) * 8 + rr;
            const int dim = kk * 16 + (mi & 1) * 8;
            uint32_t b0, b1, b2, b3;
            ldsm_x4(ks + key * pitch + dim * 2, b0, b1, b2, b3);
            mma16816(sfr[nt], a, b0, b1);
            mma16816(sfr[nt + 1], a, b2, b3);
        }
    }
}

// O[16 x DV] += P[16 x 32] V[32 x DV] for the warp's 32 keys staged at `vs`
// (pitch DV*2+16); P given in accumulator layout (fp32), converted to bf16 A
// fragments (two n-tiles of S form one k-step of P)
template <int DV>
__device__ __forceinline__ void warp_pv(const float (&pf)[4][4], uint32_t vs, float (&o)[DV / 8][4]) {
    const int lane = threadIdx.x & 31;
    constexpr int pitch = DV * 2 + 16;
    const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        uint32_t a[4];
        a[0] = pack_bf16x2(pf[2 * kk][0], pf[2 * kk][1]);
        a[1] = pack_bf16x2(pf[2 * kk][2], pf[2 * kk][3]);
        a[2] = pack_bf16x2(pf[2 * kk + 1][0], pf[2 * kk + 1][1]);
        a[3] = pack_bf16x2(pf[2 * kk + 1][2], pf[2 * kk + 1][3]);
#pragma unroll
        for (int nt = 0; nt < DV / 8; nt += 2) {
            // ldmatrix x4 .trans: matrices (keys 16kk..+7, ch 8nt..), (keys +8, ch 8nt..),
            // (keys 16kk.., ch 8nt+8..), (keys +8, ch 8nt+8..)
            const int key = kk * 16 + (mi & 1) * 8 + rr;
            const int ch = nt * 8 + (mi >> 1) * 8;
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vs + key * pitch + ch * 2, b0, b1, b2, b3);
            mma16816(o[nt], a, b0, b1);
            mma16816(o[nt + 1], a, b2, b3);
        }
    }
}


}  // namespace nsa
