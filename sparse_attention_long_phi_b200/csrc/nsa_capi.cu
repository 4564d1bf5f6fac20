// nsa_capi.cu -- libnsa: the C ABI declared in include/nsa.h.
//
// Host side only: argument validation, workspace carving, TMA descriptor
// encoding and kernel launches on the caller's stream.  Every step of the
// operator runs in the kernels included below; nothing here touches tensor
// data.  The whole library is one translation unit so that the device error
// word is shared by every kernel.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/nsa.h"
#include "k_attn_packed.cuh"
#include "k_attn_sel.cuh"
#include "k_decode.cuh"
#include "k_backward.cuh"
#include "k_bwd_kv.cuh"
#include "k_bwd_q.cuh"
#include "k_bwd_qsel.cuh"
#include "k_phi.cuh"
#include "k_topn.cuh"
#include "k_append.cuh"
#include "k_phi_grad.cuh"
#include "k_phi_bwd.cuh"

using namespace nsa;

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool encode_fn() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode != nullptr;
}

// bf16 tiled map with 128-byte swizzle (box inner extent must be 64 elements)
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
              const uint64_t* strides, const uint32_t* box) {
    if (!encode_fn()) return false;
    cuuint64_t gd[5], gs[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        gd[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
        if (i < rank - 1) gs[i] = strides[i];
    }
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
                          gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}


// ---------------------------------------------------------- launch timing
struct ProfRec {
    const char* name;
    cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof_recs;
std::vector<cudaEvent_t> g_prof_pool;

cudaEvent_t prof_event() {
    if (!g_prof_pool.empty()) {
        cudaEvent_t e = g_prof_pool.back();
        g_prof_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// brackets the launches in its scope with events on `st` when timing is on
struct ProfScope {
    const char* name;
    cudaStream_t st;
    cudaEvent_t a = nullptr, b = nullptr;
    ProfScope(const char* n, cudaStream_t s) : name(n), st(s) {
        if (!g_prof_on) return;
        std::lock_guard<std::mutex> lk(g_prof_mu);
        a = prof_event();
        b = prof_event();
        cudaEventRecord(a, st);
    }
    ~ProfScope() {
        if (!a) return;
        cudaEventRecord(b, st);
        std::lock_guard<std::mutex> lk(g_prof_mu);
        g_prof_recs.push_back({name, a, b});
    }
};

#define NSA_LAUNCH(name, st, ...)        \
    do {                                 \
        ProfScope _prof_scope(name, st); \
        __VA_ARGS__;                     \
    } while (0)

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream finishes; it reads that kernel's results
// only after griddepcontrol.wait (dep_wait()).
template <typename... KArgs, typename... Args>
nsa_status_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? NSA_OK : NSA_ERR_CUDA;
}

struct Shape {
    int64_t B, T, H, G, DK, DV, HG, l, d, lp, n, fi, fl, w;
    int64_t C, Cp, Tp, DVP, NS, NSp;
    int phi;
    float scale;
};

nsa_status_t derive(const nsa_config_t* c, Shape& s) {
    if (!c) return NSA_ERR_INVALID_ARG;
    s.B = c->batch;
    s.T = c->seqlen;
    s.H = c->num_q_heads;
    s.G = c->num_kv_groups;
    s.DK = c->d_k;
    s.DV = c->d_v;
    s.l = c->cmp_block;
    s.d = c->cmp_stride;
    s.lp = c->sel_block;
    s.n = c->sel_count;
    s.fi = c->forced_initial;
    s.fl = c->forced_local;
    s.w = c->window;
    s.phi = c->phi;
    if (s.B <= 0 || s.T <= 0 || s.H <= 0 || s.G <= 0 || s.DK <= 0 || s.DV <= 0) return NSA_ERR_INVALID_ARG;
    if (s.H % s.G) return NSA_ERR_INVALID_ARG;
    if (s.l <= 0 || s.d <= 0 || s.lp <= 0 || s.w <= 0 || s.n <= 0) return NSA_ERR_INVALID_ARG;
    if (s.l % s.d || s.lp % s.d || s.l > s.lp) return NSA_ERR_INVALID_ARG;
    if (s.fi < 0 || s.fl < 0 || s.n < s.fi + s.fl) return NSA_ERR_INVALID_ARG;
    if (c->phi != NSA_PHI_MEAN && c->phi != NSA_PHI_LINEAR) return NSA_ERR_INVALID_ARG;
    if (c->score_map != 0 && c->score_map != 1) return NSA_ERR_INVALID_ARG;
    if (!(c->scale >= 0.f)) return NSA_ERR_INVALID_ARG;
    s.HG = s.H / s.G;
    s.scale = c->scale > 0.f ? c->scale : 1.0f / std::sqrt((float)s.DK);
    s.C = s.T >= s.l ? (s.T - s.l) / s.d + 1 : 0;
    s.Cp = ceil_div(std::max<int64_t>(s.C, 1), 8) * 8;
    s.Tp = ceil_div(s.T, 8) * 8;
    s.DVP = std::max<int64_t>(s.DV, 128);
    s.NS = ceil_div(s.T, s.lp);
    s.NSp = ceil_div(s.NS, 4) * 4;
    return NSA_OK;
}

// kernels exist for these sizes only
nsa_status_t supported(const Shape& s) {
    const bool dims = (s.DK == 64 && s.DV == 64 && s.HG == 4) || (s.DK == 192 && s.DV == 128 && s.HG == 16);
    if (!dims) return NSA_ERR_UNSUPPORTED;
    if (s.lp != 64 || s.n > 16) return NSA_ERR_UNSUPPORTED;
    const int64_t cps = s.l / s.d, spb = s.lp / s.d;
    const bool blk = (cps == 2 && spb == 4) || (cps == 1 && spb == 1) || (cps == 1 && spb == 4) ||
                     (cps == 2 && spb == 2);
    if (!blk) return NSA_ERR_UNSUPPORTED;
    if (s.T > 131072 || s.B * s.T * s.H > (int64_t)1 << 31) return NSA_ERR_UNSUPPORTED;
    return NSA_OK;
}

struct FwdWs {
    size_t off_kc, off_vct, off_vt, off_bias, off_lse, off_ps, off_fix, off_vt_win, total;
};

// phi fix-up list: two counters (K, V), then one entry per K~ and V~ element
inline size_t fix_bytes(const Shape& s) {
    return 256 + (size_t)s.B * std::max<int64_t>(s.C, 1) * s.G * (s.DK + s.DV) * 4;
}

FwdWs fwd_layout(const Shape& s) {
    FwdWs w{};
    size_t o = 0;
    w.off_kc = o;
    o = align256(o + (size_t)s.B * std::max<int64_t>(s.C, 1) * s.G * s.DK * 2);
    w.off_vct = o;
    o = align256(o + (size_t)s.B * s.G * s.DV * s.Cp * 2);
    w.off_vt = o;
    o = align256(o + (size_t)s.B * s.G * s.DVP * s.Tp * 2);
    w.off_bias = o;
    o = align256(o + (size_t)(s.DK + s.DV) * 8);
    w.off_lse = o;
    o = align256(o + (size_t)s.B * s.T * s.H * 4);
    w.off_ps = o;
    o = align256(o + (size_t)s.B * s.T * s.G * s.NSp * 4);
    w.off_fix = o;
    o = align256(o + fix_bytes(s));
    w.off_vt_win = o;                 // used only when the window has its own values
    w.total = o;
    return w;
}

// forward with independent keys/values per branch: a second transposed v
inline size_t fwd_branches_total(const Shape& s) {
    return fwd_layout(s).total + align256((size_t)s.B * s.G * s.DVP * s.Tp * 2);
}

inline nsa_status_t last_launch() {
    return cudaGetLastError() == cudaSuccess ? NSA_OK : NSA_ERR_CUDA;
}

#define NSA_TRY(x)                              \
    do {                                        \
        nsa_status_t _st = (x);                 \
        if (_st != NSA_OK) return _st;          \
    } while (0)

template <typename K>
nsa_status_t set_smem(K kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
                   cudaSuccess
               ? NSA_OK
               : NSA_ERR_CUDA;
}

// ------------------------------------------------------------------- phi
template <int D>
nsa_status_t launch_phi_linear(const Shape& s, const void* x, const void* W, const void* E,
                               const double* bias, void* y, void* yT, uint32_t* fix_list,
                               unsigned int* fix_count, cudaStream_t st) {
    CUtensorMap mA, mW;
    const uint64_t dA[5] = {(uint64_t)D, (uint64_t)s.G, (uint64_t)s.d, (uint64_t)(s.T / s.d), (uint64_t)s.B};
    const uint64_t sA[4] = {(uint64_t)D * 2, (uint64_t)s.G * D * 2, (uint64_t)s.d * s.G * D * 2,
                            (uint64_t)s.T * s.G * D * 2};
    const uint32_t bA[5] = {64, 1, 1, 128, 1};
    const uint64_t dW[2] = {(uint64_t)s.l * D, (uint64_t)D};
    const uint64_t sW[1] = {(uint64_t)s.l * D * 2};
    const uint32_t bW[2] = {64, (uint32_t)(D / 2)};
    if (!make_map(&mA, x, 5, dA, sA, bA) || !make_map(&mW, W, 2, dW, sW, bW)) return NSA_ERR_CUDA;
    NSA_TRY(set_smem(phi_linear_kernel<D>, PhiGemmCfg<D>::kSmem));
    dim3 grid((unsigned)ceil_div(s.C, 128), (unsigned)(2 * s.G), (unsigned)s.B);
    NSA_LAUNCH("phi_linear_kernel", st, phi_linear_kernel<D><<<grid, 192, PhiGemmCfg<D>::kSmem, st>>>(
        mA, mW, bias, (int)s.l, (int)s.d, (int)s.C, (int)s.Cp, (int)s.G,
        reinterpret_cast<__nv_bfloat16*>(y), reinterpret_cast<__nv_bfloat16*>(yT), fix_list, fix_count));
    NSA_TRY(last_launch());
    NSA_LAUNCH("phi_fixup_kernel", st, phi_fixup_kernel<D><<<148 * 4, 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(x), reinterpret_cast<const __nv_bfloat16*>(W), bias,
        (int)s.T, (int)s.G, (int)s.l, (int)s.d, (int)s.C,
        (int)s.Cp, fix_list, fix_count, reinterpret_cast<__nv_bfloat16*>(y),
        reinterpret_cast<__nv_bfloat16*>(yT)));
    return last_launch();
}

// K~ -> kc [B,C,G,DK]; V~ -> vcT [B,G,DV,Cp] (+ vc [B,C,G,DV] if given)
nsa_status_t run_phi(const Shape& s, const void* k, const void* v, const nsa_phi_params_t* phi,
                     void* kc, void* vc, void* vcT, double* bias, uint8_t* fix, cudaStream_t st) {
    if (s.C == 0) return NSA_OK;
    if (s.phi == NSA_PHI_MEAN) {
        dim3 grid((unsigned)s.C, (unsigned)s.G, (unsigned)s.B);
        NSA_LAUNCH("phi_mean_kernel", st, phi_mean_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(k), (int)s.T,
                                              (int)s.G, (int)s.DK, (int)s.l, (int)s.d, (int)s.C,
                                              (int)s.Cp, reinterpret_cast<__nv_bfloat16*>(kc), nullptr));
        NSA_TRY(last_launch());
        NSA_LAUNCH("phi_mean_kernel", st, phi_mean_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(v), (int)s.T,
                                              (int)s.G, (int)s.DV, (int)s.l, (int)s.d, (int)s.C,
                                              (int)s.Cp, reinterpret_cast<__nv_bfloat16*>(vc),
                                              reinterpret_cast<__nv_bfloat16*>(vcT)));
        return last_launch();
    }
    if (!phi || !phi->w_k || !phi->e_k || !phi->w_v || !phi->e_v) return NSA_ERR_INVALID_ARG;
    if (!aligned16(phi->w_k) || !aligned16(phi->w_v)) return NSA_ERR_INVALID_ARG;
    NSA_LAUNCH("phi_bias_kernel", st, phi_bias_kernel<<<(unsigned)s.DK, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(phi->w_k),
                                                    reinterpret_cast<const __nv_bfloat16*>(phi->e_k),
                                                    (int)(s.l * s.DK), bias));
    NSA_TRY(last_launch());
    NSA_LAUNCH("phi_bias_kernel", st, phi_bias_kernel<<<(unsigned)s.DV, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(phi->w_v),
                                                    reinterpret_cast<const __nv_bfloat16*>(phi->e_v),
                                                    (int)(s.l * s.DV), bias + s.DK));
    NSA_TRY(last_launch());
    unsigned int* cnt = reinterpret_cast<unsigned int*>(fix);
    uint32_t* lk = reinterpret_cast<uint32_t*>(fix + 256);
    uint32_t* lv = lk + (size_t)s.B * s.C * s.G * s.DK;
    if (cudaMemsetAsync(cnt, 0, 8, st) != cudaSuccess) return NSA_ERR_CUDA;
    if (s.DK == 192) {
        NSA_TRY(launch_phi_linear<192>(s, k, phi->w_k, phi->e_k, bias, kc, nullptr, lk, cnt, st));
        return launch_phi_linear<128>(s, v, phi->w_v, phi->e_v, bias + s.DK, vc, vcT, lv, cnt + 1, st);
    }
    NSA_TRY(launch_phi_linear<64>(s, k, phi->w_k, phi->e_k, bias, kc, nullptr, lk, cnt, st));
    return launch_phi_linear<64>(s, v, phi->w_v, phi->e_v, bias + s.DK, vc, vcT, lv, cnt + 1, st);
}

// Failure-detection self-test: lane 0 waits, through the same bounded wait
// every kernel uses, on an mbarrier on which nothing ever arrives.  The wait
// expires after limit_ns, records its site in the device error word and the
// kernel returns; the other lanes return at once (no CTA barrier follows).
constexpr unsigned kSiteSelftest = 0x7F0;
__global__ void timeout_selftest_kernel(unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    (void)mbar_wait_for(&bar, 0, kSiteSelftest, limit_ns);
}

__global__ void cmp_empty_kernel(float* out, float* lse, long long rows, int DV) {
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < rows * DV) out[i] = 0.f;
    if (lse && i < rows) lse[i * 3] = -INFINITY;
}

// ----------------------------------------------------------- attention
int device_sm_count();   // SMs of the current device (decode section)

template <int DK, int DV, int HG, int MODE, int CPS, int SPB>
nsa_status_t launch_packed(const Shape& s, const CUtensorMap& mQ, const CUtensorMap& mK,
                           const CUtensorMap& mV, const PackedParams& p, cudaStream_t st) {
    using Cfg = PackedCfg<DK, DV, HG, MODE>;
    auto kern = attn_packed_kernel<DK, DV, HG, MODE, CPS, SPB>;
    const char* kern_name = MODE == kModeLse ? "attn_cmp_lse" : MODE == kModeCmp ? "attn_cmp_pv_scores" : "attn_window";
    NSA_TRY(set_smem(kern, Cfg::kSmem));
    dim3 grid((unsigned)p.n_ctas, (unsigned)s.G, (unsigned)s.B);
    if (MODE != kModeLse) {
        // persistent: one CTA per SM walks the (tile pair, group, batch) items, so that one
        // item's epilogue overlaps the next item's loads and products
        const int64_t items = (int64_t)p.n_ctas * s.G * s.B;
        grid = dim3((unsigned)std::min<int64_t>(items, device_sm_count()), 1, 1);
    }
    NSA_LAUNCH(kern_name, st, kern<<<grid, Cfg::kThreads, Cfg::kSmem, st>>>(mQ, mK, mV, p));
    return last_launch();
}

template <int DK, int DV, int HG, int MODE>
nsa_status_t launch_packed_blk(const Shape& s, const CUtensorMap& mQ, const CUtensorMap& mK,
                               const CUtensorMap& mV, const PackedParams& p, cudaStream_t st) {
    const int64_t cps = s.l / s.d, spb = s.lp / s.d;
    if (MODE != kModeCmp) return launch_packed<DK, DV, HG, MODE, 2, 4>(s, mQ, mK, mV, p, st);
    if (cps == 2 && spb == 4) return launch_packed<DK, DV, HG, MODE, 2, 4>(s, mQ, mK, mV, p, st);
    if (cps == 1 && spb == 1) return launch_packed<DK, DV, HG, MODE, 1, 1>(s, mQ, mK, mV, p, st);
    if (cps == 1 && spb == 4) return launch_packed<DK, DV, HG, MODE, 1, 4>(s, mQ, mK, mV, p, st);
    if (cps == 2 && spb == 2) return launch_packed<DK, DV, HG, MODE, 2, 2>(s, mQ, mK, mV, p, st);
    return NSA_ERR_UNSUPPORTED;
}

// Tensor maps of the attention kernels: q (packed query tiles and per-token
// head boxes), raw keys of the selected and window branches, compressed keys,
// and the transposed value copies (the K-major B operands of the P.V products).
struct AttnMaps {
    CUtensorMap mQ, mQs, mKc, mVc, mK, mVT, mVTs, mKw;
};

template <int DK, int DV, int HG>
nsa_status_t attn_maps(const Shape& s, const void* q, const void* k_slc, const void* k_win, const void* kc,
                       const void* vcT, const void* vT, const void* vTw, AttnMaps& m) {
    const uint64_t dQ[4] = {(uint64_t)s.DK, (uint64_t)s.H, (uint64_t)s.T, (uint64_t)s.B};
    const uint64_t sQ[3] = {(uint64_t)s.DK * 2, (uint64_t)s.H * s.DK * 2, (uint64_t)s.T * s.H * s.DK * 2};
    const uint32_t bQ[4] = {64, (uint32_t)HG, (uint32_t)(128 / HG), 1};
    const uint32_t bQs[4] = {64, 16, 1, 1};
    const uint64_t dK[4] = {(uint64_t)s.DK, (uint64_t)s.G, (uint64_t)s.T, (uint64_t)s.B};
    const uint64_t sK[3] = {(uint64_t)s.DK * 2, (uint64_t)s.G * s.DK * 2, (uint64_t)s.T * s.G * s.DK * 2};
    const uint32_t bK[4] = {64, 1, 64, 1};
    const uint64_t dVT[4] = {(uint64_t)s.T, (uint64_t)s.DVP, (uint64_t)s.G, (uint64_t)s.B};
    const uint64_t sVT[3] = {(uint64_t)s.Tp * 2, (uint64_t)s.DVP * s.Tp * 2, (uint64_t)s.G * s.DVP * s.Tp * 2};
    const uint32_t bVT[4] = {64, (uint32_t)s.DV, 1, 1};
    const uint32_t bVTs[4] = {64, 128, 1, 1};
    if (!make_map(&m.mQ, q, 4, dQ, sQ, bQ) || !make_map(&m.mQs, q, 4, dQ, sQ, bQs) ||
        !make_map(&m.mK, k_slc, 4, dK, sK, bK) || !make_map(&m.mKw, k_win, 4, dK, sK, bK) ||
        !make_map(&m.mVT, vTw, 4, dVT, sVT, bVT) || !make_map(&m.mVTs, vT, 4, dVT, sVT, bVTs))
        return NSA_ERR_CUDA;
    if (s.C > 0) {
        const uint64_t dKc[4] = {(uint64_t)s.DK, (uint64_t)s.G, (uint64_t)s.C, (uint64_t)s.B};
        const uint64_t sKc[3] = {(uint64_t)s.DK * 2, (uint64_t)s.G * s.DK * 2, (uint64_t)s.C * s.G * s.DK * 2};
        const uint64_t dVc[4] = {(uint64_t)s.C, (uint64_t)s.DV, (uint64_t)s.G, (uint64_t)s.B};
        const uint64_t sVc[3] = {(uint64_t)s.Cp * 2, (uint64_t)s.DV * s.Cp * 2, (uint64_t)s.G * s.DV * s.Cp * 2};
        const uint32_t bVc[4] = {64, (uint32_t)s.DV, 1, 1};
        if (!make_map(&m.mKc, kc, 4, dKc, sKc, bK) || !make_map(&m.mVc, vcT, 4, dVc, sVc, bVc))
            return NSA_ERR_CUDA;
    }
    return NSA_OK;
}

template <int HG>
PackedParams packed_params(const Shape& s, const float* gates, float* out, float* lse, float* lse_cmp,
                           float* pscore) {
    PackedParams pp{};
    pp.B = (int)s.B;
    pp.T = (int)s.T;
    pp.H = (int)s.H;
    pp.G = (int)s.G;
    pp.l = (int)s.l;
    pp.d = (int)s.d;
    pp.lp = (int)s.lp;
    pp.w = (int)s.w;
    pp.scale_log2 = s.scale * kLog2e;
    pp.gates = gates;
    pp.out = out;
    pp.lse_user = lse;
    pp.lse_cmp = lse_cmp;
    pp.pscore = pscore;
    pp.NSp = (int)s.NSp;
    pp.n_ctas = (int)ceil_div(s.T, 2 * (128 / HG));
    return pp;
}

// compressed branch: out = g_cmp o_cmp (stored), lse[..., 0], the score table;
// with obranch, o_cmp itself too
template <int DK, int DV, int HG>
nsa_status_t launch_cmp(const Shape& s, const AttnMaps& m, const float* gates, float* out, float* lse,
                        float* lse_cmp, float* pscore, cudaStream_t st, float* obranch = nullptr) {
    if (s.C > 0) {
        PackedParams pp = packed_params<HG>(s, gates, out, lse, lse_cmp, pscore);
        pp.obranch = obranch;
        NSA_TRY((launch_packed_blk<DK, DV, HG, kModeLse>(s, m.mQ, m.mKc, m.mVc, pp, st)));
        return launch_packed_blk<DK, DV, HG, kModeCmp>(s, m.mQ, m.mKc, m.mVc, pp, st);
    }
    const long long rows = s.B * s.T * s.H;
    if (obranch && cudaMemsetAsync(obranch, 0, (size_t)rows * s.DV * 4, st) != cudaSuccess) return NSA_ERR_CUDA;
    NSA_LAUNCH("cmp_empty_kernel", st, cmp_empty_kernel<<<(unsigned)ceil_div(rows * s.DV, 256), 256, 0, st>>>(out, lse, rows, (int)s.DV));
    return last_launch();
}

// selected branch under sel_idx: out += g_slc o_slc, lse[..., 1]; with obranch, o_slc too
template <int DK, int DV, int HG>
nsa_status_t launch_sel(const Shape& s, const AttnMaps& m, const float* gates, float* out, float* lse,
                        const int32_t* sel_idx, cudaStream_t st, float* obranch = nullptr) {
    SelParams sp{};
    sp.B = (int)s.B;
    sp.T = (int)s.T;
    sp.H = (int)s.H;
    sp.G = (int)s.G;
    sp.n = (int)s.n;
    sp.scale_log2 = s.scale * kLog2e;
    sp.idx = sel_idx;
    sp.gates = gates;
    sp.out = out;
    sp.obranch = obranch;
    sp.lse_user = lse;
    int64_t tpc = (s.B * s.T * s.G) / (148 * 8);
    sp.tpc = (int)std::min<int64_t>(64, std::max<int64_t>(4, tpc));
    using Cfg = SelCfg<DK, DV>;
    NSA_TRY(set_smem(attn_sel_kernel<DK, DV, HG>, Cfg::kSmem));
    sp.nchunks = (int)ceil_div(s.T, sp.tpc);
    dim3 grid((unsigned)(sp.nchunks * s.G), 1, (unsigned)s.B);
    NSA_LAUNCH("attn_sel_kernel", st, attn_sel_kernel<DK, DV, HG><<<grid, Cfg::kThreads, Cfg::kSmem, st>>>(m.mQs, m.mK, m.mVTs, sp));
    return last_launch();
}

// sliding window: out += g_win o_win, lse[..., 2]; with obranch, o_win too
template <int DK, int DV, int HG>
nsa_status_t launch_win(const Shape& s, const AttnMaps& m, const float* gates, float* out, float* lse,
                        cudaStream_t st, float* obranch = nullptr) {
    PackedParams pp = packed_params<HG>(s, gates, out, lse, nullptr, nullptr);
    pp.obranch = obranch;
    return launch_packed_blk<DK, DV, HG, kModeWin>(s, m.mQ, m.mKw, m.mVT, pp, st);
}

// Keys and values of the three branches (page 2, 滑动窗口: the branches may
// have independent keys and values).  The compressed branch compresses
// (k_cmp, v_cmp); the selected branch reads (k_slc, v_slc) and the window
// (k_win, v_win).  nsa_forward passes one k/v to all three.
struct BranchKV {
    const void *k_cmp, *v_cmp, *k_slc, *v_slc, *k_win, *v_win;
};

// obranch (optional): [3][B,T,H,DV], each branch's own output o_c before its
// gate, in the order compressed, selected, window (what the backward's
// statistics need, saved by a training forward)
template <int DK, int DV, int HG>
nsa_status_t forward_impl(const Shape& s, const void* q, const BranchKV& kv,
                          const float* gates, const nsa_phi_params_t* phi, float* out,
                          int32_t* sel_idx, float* lse, void* kc_out, void* vc_out, uint8_t* ws,
                          cudaStream_t st, float* obranch = nullptr) {
    const size_t ob_stride = (size_t)s.B * s.T * s.H * s.DV;
    float* ob_cmp = obranch;
    float* ob_slc = obranch ? obranch + ob_stride : nullptr;
    float* ob_win = obranch ? obranch + 2 * ob_stride : nullptr;
    const FwdWs L = fwd_layout(s);
    void* kc = kc_out ? kc_out : ws + L.off_kc;
    void* vcT = ws + L.off_vct;
    void* vT = ws + L.off_vt;
    const bool own_win_v = kv.v_win != kv.v_slc;
    void* vTw = own_win_v ? ws + L.off_vt_win : vT;
    double* bias = reinterpret_cast<double*>(ws + L.off_bias);
    float* lse_cmp = reinterpret_cast<float*>(ws + L.off_lse);
    float* pscore = reinterpret_cast<float*>(ws + L.off_ps);

    // 1. token compression
    NSA_TRY(run_phi(s, kv.k_cmp, kv.v_cmp, phi, kc, vc_out, vcT, bias, ws + L.off_fix, st));
    // 2. v transposed for the P.V products of the selected and window branches
    for (int pass = 0; pass < (own_win_v ? 2 : 1); ++pass) {
        dim3 grid((unsigned)ceil_div(s.Tp, 64), (unsigned)s.G, (unsigned)s.B);
        NSA_LAUNCH("transpose_v_kernel", st, transpose_v_kernel<<<grid, dim3(64, 4), 0, st>>>(
            reinterpret_cast<const __nv_bfloat16*>(pass ? kv.v_win : kv.v_slc), (int)s.T, (int)s.G, (int)s.DV,
            (int)s.DVP, (int)s.Tp, reinterpret_cast<__nv_bfloat16*>(pass ? vTw : vT)));
        NSA_TRY(last_launch());
    }
    AttnMaps m;
    NSA_TRY((attn_maps<DK, DV, HG>(s, q, kv.k_slc, kv.k_win, kc, vcT, vT, vTw, m)));
    // 3-4. compressed attention: LSE pass, then P.V~ with importance scores
    NSA_TRY((launch_cmp<DK, DV, HG>(s, m, gates, out, lse, lse_cmp, pscore, st, ob_cmp)));
    // 5. top-n selection
    {
        const long long items = s.B * s.T * s.G;
        const unsigned grid = (unsigned)ceil_div(items, 8);
        if (s.NSp <= 32 * 32) {   // rows of at most 1024 blocks: 32 candidates per lane
            NSA_LAUNCH("topn_kernel", st, topn_kernel<32><<<grid, 256, 0, st>>>(pscore, items, (int)s.T, (int)s.G,
                                                                   (int)s.NSp, (int)s.n, (int)s.lp,
                                                                   (int)s.fi, (int)s.fl, sel_idx));
        } else {
            NSA_LAUNCH("topn_kernel", st, topn_kernel<kTopnPerLane><<<grid, 256, 0, st>>>(pscore, items, (int)s.T, (int)s.G,
                                                                   (int)s.NSp, (int)s.n, (int)s.lp,
                                                                   (int)s.fi, (int)s.fl, sel_idx));
        }
        NSA_TRY(last_launch());
    }
    // 6. selected attention
    NSA_TRY((launch_sel<DK, DV, HG>(s, m, gates, out, lse, sel_idx, st, ob_slc)));
    // 7. sliding window
    return launch_win<DK, DV, HG>(s, m, gates, out, lse, st, ob_win);
}


// ---------------------------------------------- linear phi backward (tcgen05)
// The products need whole 256-column tiles of the l*D inputs.
bool phi_bwd_tensor_ok(const Shape& s) { return (s.l * s.DK) % 256 == 0 && (s.l * s.DV) % 256 == 0; }

// kPhiT: dX[b, i*d + j, g, :] += (dY[b,i,g,:] W)[j*D ..]; kPhiDW: dW = dY^T X + s E
template <int D, int MODE>
nsa_status_t launch_phi_bwd(const Shape& s, const void* dyb, const void* src, float* dX, float* dW,
                            const float* colsum, const void* E, cudaStream_t st) {
    CUtensorMap mY, mB;
    const uint64_t dY[4] = {(uint64_t)D, (uint64_t)s.G, (uint64_t)s.C, (uint64_t)s.B};
    const uint64_t sY[3] = {(uint64_t)D * 2, (uint64_t)s.G * D * 2, (uint64_t)s.C * s.G * D * 2};
    const uint32_t bY[4] = {64, 1, MODE == kPhiT ? 128u : 64u, 1};
    if (!make_map(&mY, dyb, 4, dY, sY, bY)) return NSA_ERR_CUDA;
    if (MODE == kPhiT) {
        const uint64_t dW2[2] = {(uint64_t)s.l * D, (uint64_t)D};
        const uint64_t sW2[1] = {(uint64_t)s.l * D * 2};
        const uint32_t bW2[2] = {64, 64};
        if (!make_map(&mB, src, 2, dW2, sW2, bW2)) return NSA_ERR_CUDA;
    } else {
        const uint64_t dX5[5] = {(uint64_t)D, (uint64_t)s.G, (uint64_t)s.d, (uint64_t)(s.T / s.d), (uint64_t)s.B};
        const uint64_t sX5[4] = {(uint64_t)D * 2, (uint64_t)s.G * D * 2, (uint64_t)s.d * s.G * D * 2,
                                 (uint64_t)s.T * s.G * D * 2};
        const uint32_t bX5[5] = {64, 1, 1, 64, 1};
        if (!make_map(&mB, src, 5, dX5, sX5, bX5)) return NSA_ERR_CUDA;
    }
    PhiBwdParams pp{};
    pp.B = (int)s.B;
    pp.T = (int)s.T;
    pp.G = (int)s.G;
    pp.C = (int)s.C;
    pp.D = D;
    pp.l = (int)s.l;
    pp.d = (int)s.d;
    pp.dX = dX;
    pp.dW = dW;
    pp.s = colsum;
    pp.E = reinterpret_cast<const __nv_bfloat16*>(E);
    NSA_TRY(set_smem(phi_bwd_gemm<MODE>, PhiBwdCfg::kSmem));
    const dim3 grid((unsigned)(s.l * D / PhiBwdCfg::NT),
                    (unsigned)(MODE == kPhiT ? ceil_div(s.C, 128) : ceil_div(D, 128)),
                    (unsigned)(MODE == kPhiT ? s.B * s.G : 1));
    NSA_LAUNCH(MODE == kPhiT ? "phi_bwd_gemm_dx" : "phi_bwd_gemm_dw", st,
               phi_bwd_gemm<MODE><<<grid, PhiBwdCfg::kThreads, PhiBwdCfg::kSmem, st>>>(mY, mB, pp));
    return last_launch();
}

// dK~ and dV~ (fp32 [B,C,G,D]) rounded to bf16 into the workspace
nsa_status_t phi_bwd_operands(const Shape& s, const float* dkc, const float* dvc, __nv_bfloat16* dyb,
                              cudaStream_t st) {
    const long long nk4 = s.B * s.C * s.G * s.DK / 4, nv4 = s.B * s.C * s.G * s.DV / 4;
    NSA_LAUNCH("f32_to_bf16_kernel", st, f32_to_bf16_kernel<<<(unsigned)ceil_div(nk4, 256), 256, 0, st>>>(dkc, dyb, nk4));
    NSA_TRY(last_launch());
    NSA_LAUNCH("f32_to_bf16_kernel", st, f32_to_bf16_kernel<<<(unsigned)ceil_div(nv4, 256), 256, 0, st>>>(
        dvc, dyb + (size_t)s.B * s.C * s.G * s.DK, nv4));
    return last_launch();
}

// -------------------------------------------------------------- backward
struct BwdWs {
    size_t off_kc, off_vc, off_vct, off_bias, off_lse2, off_dlt, off_dkc, off_dvc, off_cnt,
        off_cur, off_off, off_choff, off_list, off_fix, off_ones, off_obuf, off_lsen, off_lsec, off_ps, off_vt,
        off_dyb, total;
};

BwdWs bwd_layout(const Shape& s) {
    BwdWs w{};
    const int64_t C1 = std::max<int64_t>(s.C, 1);
    const int64_t NE = s.B * s.G * s.NS;
    size_t o = 0;
    w.off_kc = o;
    o = align256(o + (size_t)s.B * C1 * s.G * s.DK * 2);
    w.off_vc = o;
    o = align256(o + (size_t)s.B * C1 * s.G * s.DV * 2);
    w.off_vct = o;
    o = align256(o + (size_t)s.B * s.G * s.DV * s.Cp * 2);
    w.off_bias = o;
    o = align256(o + (size_t)(s.DK + s.DV) * 8);
    w.off_lse2 = o;
    o = align256(o + (size_t)s.B * s.T * s.H * 3 * 4);
    w.off_dlt = o;
    o = align256(o + (size_t)s.B * s.T * s.H * 3 * 4);
    w.off_dkc = o;
    o = align256(o + (size_t)s.B * C1 * s.G * s.DK * 4);
    w.off_dvc = o;
    o = align256(o + (size_t)s.B * C1 * s.G * s.DV * 4);
    w.off_cnt = o;
    o = align256(o + (size_t)NE * 4);
    w.off_cur = o;
    o = align256(o + (size_t)NE * 4);
    w.off_off = o;
    o = align256(o + (size_t)(NE + 1) * 4);
    w.off_choff = o;
    o = align256(o + (size_t)(NE + 1) * 4);
    w.off_list = o;
    o = align256(o + (size_t)s.B * s.T * s.G * s.n * 4);
    w.off_fix = o;
    o = align256(o + fix_bytes(s));
    // per-branch statistics through the forward kernels
    w.off_ones = o;
    o = align256(o + (size_t)s.B * s.T * s.H * 3 * 4);
    w.off_obuf = o;
    o = align256(o + (size_t)s.B * s.T * s.H * s.DV * 4);
    w.off_lsen = o;
    o = align256(o + (size_t)s.B * s.T * s.H * 3 * 4);
    w.off_lsec = o;
    o = align256(o + (size_t)s.B * s.T * s.H * 4);
    w.off_ps = o;
    o = align256(o + (size_t)s.B * s.T * s.G * s.NSp * 4);
    w.off_vt = o;
    o = align256(o + (size_t)s.B * s.G * s.DVP * s.Tp * 2);
    // bf16 copies of dK~ and dV~ for the linear phi's tensor-core products
    w.off_dyb = o;
    o = align256(o + (size_t)s.B * C1 * s.G * (s.DK + s.DV) * 2);
    w.total = o;
    return w;
}

template <int DK, int DV>
nsa_status_t backward_impl(const Shape& s, const void* q, const void* k, const void* v,
                           const float* gates, const nsa_phi_params_t* phi, const void* dout,
                           const int32_t* sel_idx, float* dq, float* dk, float* dv, float* dgates,
                           uint8_t* ws, cudaStream_t st, const float* saved_lse = nullptr,
                           const float* saved_o = nullptr) {
    const BwdWs L = bwd_layout(s);
    const int64_t NE = s.B * s.G * s.NS;
    BwdParams p{};
    p.B = (int)s.B;
    p.T = (int)s.T;
    p.H = (int)s.H;
    p.G = (int)s.G;
    p.HG = (int)s.HG;
    p.DK = DK;
    p.DV = DV;
    p.l = (int)s.l;
    p.d = (int)s.d;
    p.lp = (int)s.lp;
    p.n = (int)s.n;
    p.w = (int)s.w;
    p.C = (int)s.C;
    p.NSb = (int)s.NS;
    p.scale = s.scale;
    p.scale_log2 = s.scale * kLog2e;
    p.q = reinterpret_cast<const __nv_bfloat16*>(q);
    p.k = reinterpret_cast<const __nv_bfloat16*>(k);
    p.v = reinterpret_cast<const __nv_bfloat16*>(v);
    p.kc = reinterpret_cast<const __nv_bfloat16*>(ws + L.off_kc);
    p.vc = reinterpret_cast<const __nv_bfloat16*>(ws + L.off_vc);
    p.dout = reinterpret_cast<const __nv_bfloat16*>(dout);
    p.wk = phi ? reinterpret_cast<const __nv_bfloat16*>(phi->w_k) : nullptr;
    p.wv = phi ? reinterpret_cast<const __nv_bfloat16*>(phi->w_v) : nullptr;
    p.gates = gates;
    p.idx = sel_idx;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.dgates = dgates;
    p.lse2 = reinterpret_cast<float*>(ws + L.off_lse2);
    p.dlt = reinterpret_cast<float*>(ws + L.off_dlt);
    p.dkc = reinterpret_cast<float*>(ws + L.off_dkc);
    p.dvc = reinterpret_cast<float*>(ws + L.off_dvc);
    p.cnt = reinterpret_cast<int*>(ws + L.off_cnt);
    p.cursor = reinterpret_cast<int*>(ws + L.off_cur);
    p.off = reinterpret_cast<int*>(ws + L.off_off);
    p.chunk_off = reinterpret_cast<int*>(ws + L.off_choff);
    p.list = reinterpret_cast<int*>(ws + L.off_list);
    p.phi = s.phi;

    // compressed keys/values of the forward (row layout)
    NSA_TRY(run_phi(s, k, v, phi, ws + L.off_kc, ws + L.off_vc, ws + L.off_vct,
                    reinterpret_cast<double*>(ws + L.off_bias), ws + L.off_fix, st));
    if (cudaMemsetAsync(dk, 0, (size_t)s.B * s.T * s.G * DK * 4, st) != cudaSuccess ||
        cudaMemsetAsync(dv, 0, (size_t)s.B * s.T * s.G * DV * 4, st) != cudaSuccess ||
        cudaMemsetAsync(ws + L.off_dkc, 0, L.off_cnt - L.off_dkc, st) != cudaSuccess ||
        cudaMemsetAsync(ws + L.off_cnt, 0, L.off_off - L.off_cnt, st) != cudaSuccess)
        return NSA_ERR_CUDA;
    // per-branch statistics under the given selection, from the forward kernels:
    // with unit gates each branch's output is its own o_c, whose dot product with
    // dO gives d(gate_c) and D_c = g_c <dO, o_c>; the kernels' LSEs come along.
    // A training forward that saved o_c and the LSEs spares these passes.
    if (saved_o) {
        const long long rows = s.B * s.T * s.H;
        NSA_LAUNCH("bwd_branch_stats", st, bwd_branch_stats3<<<(unsigned)ceil_div(rows, 8), 256, 0, st>>>(
            saved_o, reinterpret_cast<const __nv_bfloat16*>(dout), gates, saved_lse, rows, DV, dgates, p.dlt, p.lse2));
        NSA_TRY(last_launch());
    } else {
        constexpr int HG = DK == 192 ? 16 : 4;
        const long long rows = s.B * s.T * s.H;
        float* ones = reinterpret_cast<float*>(ws + L.off_ones);
        float* obuf = reinterpret_cast<float*>(ws + L.off_obuf);
        float* lsen = reinterpret_cast<float*>(ws + L.off_lsen);
        void* vT = ws + L.off_vt;
        NSA_LAUNCH("fill_f32", st, fill_f32<<<(unsigned)ceil_div(rows * 3, 256), 256, 0, st>>>(ones, rows * 3, 1.f));
        NSA_TRY(last_launch());
        dim3 tg((unsigned)ceil_div(s.Tp, 64), (unsigned)s.G, (unsigned)s.B);
        NSA_LAUNCH("transpose_v_kernel", st, transpose_v_kernel<<<tg, dim3(64, 4), 0, st>>>(
            reinterpret_cast<const __nv_bfloat16*>(v), (int)s.T, (int)s.G, (int)s.DV, (int)s.DVP, (int)s.Tp,
            reinterpret_cast<__nv_bfloat16*>(vT)));
        NSA_TRY(last_launch());
        AttnMaps m;
        NSA_TRY((attn_maps<DK, DV, HG>(s, q, k, k, ws + L.off_kc, ws + L.off_vct, vT, vT, m)));
        const size_t obytes = (size_t)rows * DV * 4;
        for (int br = 0; br < 3; ++br) {
            if (br == 0) {
                NSA_TRY((launch_cmp<DK, DV, HG>(s, m, ones, obuf, lsen, reinterpret_cast<float*>(ws + L.off_lsec),
                                                reinterpret_cast<float*>(ws + L.off_ps), st)));
            } else {
                if (cudaMemsetAsync(obuf, 0, obytes, st) != cudaSuccess) return NSA_ERR_CUDA;
                if (br == 1) NSA_TRY((launch_sel<DK, DV, HG>(s, m, ones, obuf, lsen, sel_idx, st)));
                else NSA_TRY((launch_win<DK, DV, HG>(s, m, ones, obuf, lsen, st)));
            }
            NSA_LAUNCH("bwd_branch_stats", st, bwd_branch_stats<<<(unsigned)ceil_div(rows, 8), 256, 0, st>>>(
                obuf, reinterpret_cast<const __nv_bfloat16*>(dout), gates, lsen, br, rows, DV, dgates, p.dlt, p.lse2));
            NSA_TRY(last_launch());
        }
    }
    // dq of the selected branch (tcgen05, per token and group, transposed products), added
    if (cudaMemsetAsync(dq, 0, (size_t)s.B * s.T * s.H * DK * 4, st) != cudaSuccess) return NSA_ERR_CUDA;
    {
        constexpr int HG = DK == 192 ? 16 : 4;
        using Cfg = BqsCfg<DK, DV>;
        CUtensorMap mQs, mOs, mK, mV;
        const uint32_t bH[4] = {64, 16, 1, 1};
        const uint32_t bKV[4] = {64, 1, 64, 1};
        const uint64_t dQ[4] = {(uint64_t)DK, (uint64_t)s.H, (uint64_t)s.T, (uint64_t)s.B};
        const uint64_t sQ[3] = {(uint64_t)DK * 2, (uint64_t)s.H * DK * 2, (uint64_t)s.T * s.H * DK * 2};
        const uint64_t dO[4] = {(uint64_t)DV, (uint64_t)s.H, (uint64_t)s.T, (uint64_t)s.B};
        const uint64_t sO[3] = {(uint64_t)DV * 2, (uint64_t)s.H * DV * 2, (uint64_t)s.T * s.H * DV * 2};
        const uint64_t dK[4] = {(uint64_t)DK, (uint64_t)s.G, (uint64_t)s.T, (uint64_t)s.B};
        const uint64_t sK[3] = {(uint64_t)DK * 2, (uint64_t)s.G * DK * 2, (uint64_t)s.T * s.G * DK * 2};
        const uint64_t dV[4] = {(uint64_t)DV, (uint64_t)s.G, (uint64_t)s.T, (uint64_t)s.B};
        const uint64_t sV[3] = {(uint64_t)DV * 2, (uint64_t)s.G * DV * 2, (uint64_t)s.T * s.G * DV * 2};
        if (!make_map(&mQs, q, 4, dQ, sQ, bH) || !make_map(&mOs, dout, 4, dO, sO, bH) ||
            !make_map(&mK, k, 4, dK, sK, bKV) || !make_map(&mV, v, 4, dV, sV, bKV))
            return NSA_ERR_CUDA;
        BqsParams qp{};
        qp.bp = p;
        const int64_t tpc = (s.B * s.T * s.G) / (148 * 8);
        qp.tpc = (int)std::min<int64_t>(64, std::max<int64_t>(4, tpc));
        qp.nchunks = (int)ceil_div(s.T, qp.tpc);
        NSA_TRY(set_smem(bwd_q_sel<DK, DV, HG>, Cfg::kSmem));
        const dim3 grid((unsigned)(qp.nchunks * s.G), 1, (unsigned)s.B);
        NSA_LAUNCH("bwd_q_sel", st, bwd_q_sel<DK, DV, HG><<<grid, Cfg::kThreads, Cfg::kSmem, st>>>(mQs, mOs, mK, mV, qp));
        NSA_TRY(last_launch());
    }
    // dq of the window and compressed branches (tcgen05, packed query tiles), added
    {
        constexpr int HG = DK == 192 ? 16 : 4;
        using Cfg = BqCfg<DK, DV>;
        CUtensorMap mQ, mO, mK, mV, mKc, mVc;
        const uint32_t bQ[4] = {64, (uint32_t)HG, (uint32_t)(128 / HG), 1};
        const uint32_t bKV[4] = {64, 1, 64, 1};
        const uint64_t dQ[4] = {(uint64_t)DK, (uint64_t)s.H, (uint64_t)s.T, (uint64_t)s.B};
        const uint64_t sQ[3] = {(uint64_t)DK * 2, (uint64_t)s.H * DK * 2, (uint64_t)s.T * s.H * DK * 2};
        const uint64_t dO[4] = {(uint64_t)DV, (uint64_t)s.H, (uint64_t)s.T, (uint64_t)s.B};
        const uint64_t sO[3] = {(uint64_t)DV * 2, (uint64_t)s.H * DV * 2, (uint64_t)s.T * s.H * DV * 2};
        const uint64_t dK[4] = {(uint64_t)DK, (uint64_t)s.G, (uint64_t)s.T, (uint64_t)s.B};
        const uint64_t sK[3] = {(uint64_t)DK * 2, (uint64_t)s.G * DK * 2, (uint64_t)s.T * s.G * DK * 2};
        const uint64_t dV[4] = {(uint64_t)DV, (uint64_t)s.G, (uint64_t)s.T, (uint64_t)s.B};
        const uint64_t sV[3] = {(uint64_t)DV * 2, (uint64_t)s.G * DV * 2, (uint64_t)s.T * s.G * DV * 2};
        if (!make_map(&mQ, q, 4, dQ, sQ, bQ) || !make_map(&mO, dout, 4, dO, sO, bQ) ||
            !make_map(&mK, k, 4, dK, sK, bKV) || !make_map(&mV, v, 4, dV, sV, bKV))
            return NSA_ERR_CUDA;
        NSA_TRY(set_smem(bwd_q_dense<DK, DV, HG, kBrWin>, Cfg::kSmem));
        NSA_TRY(set_smem(bwd_q_dense<DK, DV, HG, kBrCmp>, Cfg::kSmem));
        const dim3 grid((unsigned)ceil_div(s.T, 128 / HG), 1, (unsigned)(s.B * s.G));
        NSA_LAUNCH("bwd_q_dense_win", st, bwd_q_dense<DK, DV, HG, kBrWin><<<grid, Cfg::kThreads, Cfg::kSmem, st>>>(mQ, mO, mK, mV, p));
        NSA_TRY(last_launch());
        if (s.C > 0) {
            const uint64_t dKc[4] = {(uint64_t)DK, (uint64_t)s.G, (uint64_t)s.C, (uint64_t)s.B};
            const uint64_t sKc[3] = {(uint64_t)DK * 2, (uint64_t)s.G * DK * 2, (uint64_t)s.C * s.G * DK * 2};
            const uint64_t dVc[4] = {(uint64_t)DV, (uint64_t)s.G, (uint64_t)s.C, (uint64_t)s.B};
            const uint64_t sVc[3] = {(uint64_t)DV * 2, (uint64_t)s.G * DV * 2, (uint64_t)s.C * s.G * DV * 2};
            if (!make_map(&mKc, ws + L.off_kc, 4, dKc, sKc, bKV) || !make_map(&mVc, ws + L.off_vc, 4, dVc, sVc, bKV))
                return NSA_ERR_CUDA;
            NSA_LAUNCH("bwd_q_dense_cmp", st, bwd_q_dense<DK, DV, HG, kBrCmp><<<grid, Cfg::kThreads, Cfg::kSmem, st>>>(mQ, mO, mKc, mVc, p));
            NSA_TRY(last_launch());
        }
    }
    // selected branch: block pairs -> the tokens that chose them (with which halves)
    const int64_t NP = ceil_div(s.NS, 2);
    const int64_t NEp = s.B * s.G * NP;
    BkvParams kp{};
    kp.bp = p;
    kp.n_pairs = (int)NP;
    kp.pcnt = p.cnt;
    kp.poff = p.off;
    kp.pchunk = p.chunk_off;
    kp.plist = p.list;
    {
        const long long rows = s.B * s.T * s.G;
        NSA_LAUNCH("bwd_pair_count", st, bwd_pair_count<<<(unsigned)ceil_div(rows, 256), 256, 0, st>>>(p, (int)NP, p.cnt));
        NSA_TRY(last_launch());
        NSA_LAUNCH("bwd_pair_scan", st, bwd_pair_scan<<<1, 1024, 0, st>>>((int)NEp, p.cnt, p.off, p.chunk_off));
        NSA_TRY(last_launch());
        NSA_LAUNCH("bwd_pair_fill", st, bwd_pair_fill<<<(unsigned)ceil_div(rows, 256), 256, 0, st>>>(p, (int)NP, p.off, p.cursor, p.list));
        NSA_TRY(last_launch());
    }
    // key-centric dK/dV of the three branches (tcgen05, 128 keys per tile)
    {
        constexpr int HG = DK == 192 ? 16 : 4;
        using Cfg = BkvCfg<DK, DV>;
        CUtensorMap mK, mV, mKc, mVc, mQ, mO;
        const uint32_t bKV[4] = {64, 1, 128, 1};
        const uint64_t dK[4] = {(uint64_t)DK, (uint64_t)s.G, (uint64_t)s.T, (uint64_t)s.B};
        const uint64_t sK[3] = {(uint64_t)DK * 2, (uint64_t)s.G * DK * 2, (uint64_t)s.T * s.G * DK * 2};
        const uint64_t dV[4] = {(uint64_t)DV, (uint64_t)s.G, (uint64_t)s.T, (uint64_t)s.B};
        const uint64_t sV[3] = {(uint64_t)DV * 2, (uint64_t)s.G * DV * 2, (uint64_t)s.T * s.G * DV * 2};
        const uint32_t bR[4] = {64, (uint32_t)HG, (uint32_t)(kBkvRows / HG), 1};
        const uint64_t dQ[4] = {(uint64_t)DK, (uint64_t)s.H, (uint64_t)s.T, (uint64_t)s.B};
        const uint64_t sQ[3] = {(uint64_t)DK * 2, (uint64_t)s.H * DK * 2, (uint64_t)s.T * s.H * DK * 2};
        const uint64_t dO[4] = {(uint64_t)DV, (uint64_t)s.H, (uint64_t)s.T, (uint64_t)s.B};
        const uint64_t sO[3] = {(uint64_t)DV * 2, (uint64_t)s.H * DV * 2, (uint64_t)s.T * s.H * DV * 2};
        if (!make_map(&mK, k, 4, dK, sK, bKV) || !make_map(&mV, v, 4, dV, sV, bKV) ||
            !make_map(&mQ, q, 4, dQ, sQ, bR) || !make_map(&mO, dout, 4, dO, sO, bR))
            return NSA_ERR_CUDA;
        NSA_TRY(set_smem(bwd_kv_tc<DK, DV, HG, kBrWin>, Cfg::kSmem));
        NSA_TRY(set_smem(bwd_kv_tc<DK, DV, HG, kBrSlc>, Cfg::kSmem));
        NSA_TRY(set_smem(bwd_kv_tc<DK, DV, HG, kBrCmp>, Cfg::kSmem));
        const unsigned bg = (unsigned)(s.B * s.G);
        dim3 gw((unsigned)ceil_div(s.T, 128), (unsigned)ceil_div(128 + s.w - 1, kBkvChunk), bg);
        NSA_LAUNCH("bwd_kv_tc_win", st, bwd_kv_tc<DK, DV, HG, kBrWin><<<gw, Cfg::kThreads, Cfg::kSmem, st>>>(mK, mV, mQ, mO, kp));
        NSA_TRY(last_launch());
        const int64_t maxch = NEp + ceil_div(s.B * s.T * s.G * s.n, kBkvChunk);
        NSA_LAUNCH("bwd_kv_tc_slc", st, bwd_kv_tc<DK, DV, HG, kBrSlc><<<(unsigned)maxch, Cfg::kThreads, Cfg::kSmem, st>>>(mK, mV, mQ, mO, kp));
        NSA_TRY(last_launch());
        if (s.C > 0) {
            const uint64_t dKc[4] = {(uint64_t)DK, (uint64_t)s.G, (uint64_t)s.C, (uint64_t)s.B};
            const uint64_t sKc[3] = {(uint64_t)DK * 2, (uint64_t)s.G * DK * 2, (uint64_t)s.C * s.G * DK * 2};
            const uint64_t dVc[4] = {(uint64_t)DV, (uint64_t)s.G, (uint64_t)s.C, (uint64_t)s.B};
            const uint64_t sVc[3] = {(uint64_t)DV * 2, (uint64_t)s.G * DV * 2, (uint64_t)s.C * s.G * DV * 2};
            if (!make_map(&mKc, ws + L.off_kc, 4, dKc, sKc, bKV) || !make_map(&mVc, ws + L.off_vc, 4, dVc, sVc, bKV))
                return NSA_ERR_CUDA;
            dim3 gc((unsigned)ceil_div(s.C, 128), (unsigned)ceil_div(s.T, kBkvChunk), bg);
            NSA_LAUNCH("bwd_kv_tc_cmp", st, bwd_kv_tc<DK, DV, HG, kBrCmp><<<gc, Cfg::kThreads, Cfg::kSmem, st>>>(mKc, mVc, mQ, mO, kp));
            NSA_TRY(last_launch());
            if (s.phi == NSA_PHI_LINEAR && phi_bwd_tensor_ok(s)) {
                __nv_bfloat16* dyb = reinterpret_cast<__nv_bfloat16*>(ws + L.off_dyb);
                NSA_TRY(phi_bwd_operands(s, p.dkc, p.dvc, dyb, st));
                NSA_TRY((launch_phi_bwd<DK, kPhiT>(s, dyb, p.wk, dk, nullptr, nullptr, nullptr, st)));
                NSA_TRY((launch_phi_bwd<DV, kPhiT>(s, dyb + (size_t)s.B * s.C * s.G * DK, p.wv, dv, nullptr,
                                                   nullptr, nullptr, st)));
            } else {
                dim3 gp((unsigned)s.T, (unsigned)s.G, (unsigned)s.B);
                NSA_LAUNCH("bwd_phiT_kernel", st, bwd_phiT_kernel<DK><<<gp, DK, 0, st>>>(p, p.dkc, p.wk, dk));
                NSA_TRY(last_launch());
                NSA_LAUNCH("bwd_phiT_kernel", st, bwd_phiT_kernel<DV><<<gp, DV, 0, st>>>(p, p.dvc, p.wv, dv));
                NSA_TRY(last_launch());
            }
        }
    }
    return NSA_OK;
}

// ---------------------------------------------------------------- decode
// SMs of the current device (cached per device)
int device_sm_count() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

template <int DK, int DV>
nsa_status_t decode_launch(DecParams& p, const Shape& s, int S, cudaStream_t st) {
    constexpr int smem = dec_stream_smem<DK, DV>(), smem3 = dec_slcwin_smem<DK, DV>();
    constexpr int smemw = dec_win_smem<DK, DV>();
    const int nsm = device_sm_count();
    // persistent streaming kernels: as many CTAs as fit on the device at once
    int occ1 = 1, occ3 = 1;
    NSA_TRY(set_smem(dec_cmp_stream<DK, DV>, smem));
    NSA_TRY(set_smem(dec_slcwin_stream<DK, DV>, smem3));
    NSA_TRY(set_smem(dec_win_stream<DK, DV>, smemw));
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ1, dec_cmp_stream<DK, DV>, 256, smem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ3, dec_slcwin_stream<DK, DV>, 256, smem3) != cudaSuccess)
        return NSA_ERR_CUDA;
    p.grid1 = std::min(kDecMaxGrid, nsm * std::max(1, occ1));
    p.grid3 = std::min(kDecMaxGrid, nsm * std::max(1, occ3));
    p.gridw = std::min(kDecMaxGrid, nsm);
    NSA_LAUNCH("dec_cmp_stream", st, dec_cmp_stream<DK, DV><<<(unsigned)p.grid1, 256, smem, st>>>(p));
    NSA_TRY(last_launch());
    // the three dependent kernels start while their predecessor drains
    const int smem2 = (p.NCH * 16 + p.NSmax) * 4;
    NSA_TRY(set_smem(dec_cmp_combine<DV>, smem2));
    NSA_LAUNCH("dec_cmp_combine", st,
               NSA_TRY(launch_dependent(dec_cmp_combine<DV>, dim3((unsigned)s.G, (unsigned)S), dim3(256), smem2, st, p)));
    // the window stream runs beside the combine (one CTA per SM next to a combine CTA)
    // and waits for it before exiting; the selected stream after it sees the selection
    NSA_LAUNCH("dec_win_stream", st,
               NSA_TRY(launch_dependent(dec_win_stream<DK, DV>, dim3((unsigned)p.gridw), dim3(kDecWinW * 32), smemw, st, p)));
    NSA_LAUNCH("dec_slcwin_stream", st,
               NSA_TRY(launch_dependent(dec_slcwin_stream<DK, DV>, dim3((unsigned)p.grid3), dim3(256), smem3, st, p)));
    NSA_LAUNCH("dec_final", st,
               NSA_TRY(launch_dependent(dec_final<DV>, dim3((unsigned)s.G, (unsigned)S, (unsigned)ceil_div(s.HG, kDecFinalHeads)), dim3(256), 0, st, p)));
    return last_launch();
}

nsa_status_t decode_impl(const Shape& s, int S, const void* q, const void* kcache, const void* vcache,
                         const int64_t* kv_off, const void* kccache, const void* vccache,
                         const int64_t* cmp_off, const float* gates, float* out, int32_t* sel_idx,
                         float* lse, uint8_t* ws, cudaStream_t st, const int64_t* kv_len = nullptr) {
    DecParams p{};
    p.S = S;
    p.H = (int)s.H;
    p.G = (int)s.G;
    p.HG = (int)s.HG;
    p.DK = (int)s.DK;
    p.DV = (int)s.DV;
    p.l = (int)s.l;
    p.d = (int)s.d;
    p.lp = (int)s.lp;
    p.n = (int)s.n;
    p.fi = (int)s.fi;
    p.fl = (int)s.fl;
    p.w = (int)s.w;
    p.spb = (int)(s.lp / s.d);
    p.cps = (int)(s.l / s.d);
    p.nbs = (31 + p.cps - 1) / p.spb + 1;
    p.scale_log2 = s.scale * kLog2e;
    p.q = reinterpret_cast<const __nv_bfloat16*>(q);
    p.kcache = reinterpret_cast<const __nv_bfloat16*>(kcache);
    p.vcache = reinterpret_cast<const __nv_bfloat16*>(vcache);
    p.kccache = reinterpret_cast<const __nv_bfloat16*>(kccache);
    p.vccache = reinterpret_cast<const __nv_bfloat16*>(vccache);
    p.kv_off = kv_off;
    p.cmp_off = cmp_off;
    p.kv_len = kv_len;
    p.gates = gates;
    p.out = out;
    p.sel_idx = sel_idx;
    p.lse = lse;
    p.Lmax = (int)s.T;
    p.Cmax = (int)(s.T >= s.l ? (s.T - s.l) / s.d + 1 : 1);
    p.NCH = (int)ceil_div(p.Cmax, 32);
    p.NSmax = (int)ceil_div(s.T, s.lp);
    // records of a pair: at most n (selected stream) and w/32 + 2 (window stream)
    if (S > kDecMaxSeqs || p.NCH > kDecMaxChunks || s.n > kDecMaxRecs || s.w / 32 + 2 > kDecMaxRecs ||
        p.nbs > kDecNBS || 32 % p.spb != 0)
        return NSA_ERR_UNSUPPORTED;
    size_t o = 0;
    auto carve = [&](size_t bytes) {
        float* r = reinterpret_cast<float*>(ws + o);
        o = align256(o + bytes);
        return r;
    };
    const size_t SG = (size_t)S * s.G;
    p.cmax = carve(SG * p.NCH * 16 * 4);
    p.bsum = carve(SG * p.NCH * kDecNBS * 16 * 4);
    p.part1 = carve((kDecMaxGrid * kDecW + SG) * 16 * (s.DV + 4) * 4);
    p.lsecmp = carve(SG * 16 * 4);
    p.part2 = carve((kDecMaxGrid * kDecW + SG) * 16 * (s.DV + 4) * 4);
    p.partw = carve((kDecMaxGrid * kDecWinW + SG) * 16 * (s.DV + 4) * 4);
    p.cpre = reinterpret_cast<int*>(carve((size_t)(S + 1) * 4));
    p.wpre = reinterpret_cast<int*>(carve((size_t)(S + 1) * 4));
    if (s.DK == 192) return decode_launch<192, 128>(p, s, S, st);
    return decode_launch<64, 64>(p, s, S, st);
}

}  // namespace

// ==================================================================== C ABI

extern "C" {

const char* nsa_status_string(nsa_status_t st) {
    switch (st) {
        case NSA_OK: return "ok";
        case NSA_ERR_INVALID_ARG: return "invalid argument";
        case NSA_ERR_UNSUPPORTED: return "unsupported configuration";
        case NSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case NSA_ERR_CUDA: return "CUDA call or kernel launch failed";
        case NSA_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait expired";
    }
    return "unknown status";
}

int64_t nsa_num_cmp_blocks(const nsa_config_t* cfg, int64_t len) {
    if (!cfg || cfg->cmp_stride <= 0 || cfg->cmp_block <= 0 || len < cfg->cmp_block) return 0;
    return (len - cfg->cmp_block) / cfg->cmp_stride + 1;
}

size_t nsa_workspace_size(const nsa_config_t* cfg, int32_t mode) {
    Shape s;
    if (derive(cfg, s) != NSA_OK) return 0;
    if (mode == NSA_MODE_FORWARD) return fwd_layout(s).total;
    if (mode == NSA_MODE_FORWARD_BRANCHES) return fwd_branches_total(s);
    if (mode == NSA_MODE_DECODE) return decode_ws_bytes(s.B, s.T, s.G, s.l, s.d, s.lp, s.w, s.n, s.DV);
    if (mode == NSA_MODE_BACKWARD) return bwd_layout(s).total;
    return 0;
}

int64_t nsa_forward_score_table(const nsa_config_t* cfg, int64_t* row_stride) {
    Shape s;
    if (derive(cfg, s) != NSA_OK) return -1;
    if (row_stride) *row_stride = s.NSp;
    return (int64_t)fwd_layout(s).off_ps;
}

nsa_status_t nsa_compress(const nsa_config_t* cfg, const void* k, const void* v,
                          const nsa_phi_params_t* phi, void* kc, void* vc, void* workspace,
                          size_t workspace_bytes, void* stream) {
    Shape s;
    NSA_TRY(derive(cfg, s));
    NSA_TRY(supported(s));
    if (!k || !v || !kc || !vc) return NSA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(kc) || !aligned16(vc)) return NSA_ERR_INVALID_ARG;
    const FwdWs L = fwd_layout(s);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return NSA_ERR_WORKSPACE;
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    return run_phi(s, k, v, phi, kc, vc, ws + L.off_vct, reinterpret_cast<double*>(ws + L.off_bias),
                   ws + L.off_fix, reinterpret_cast<cudaStream_t>(stream));
}

nsa_status_t nsa_forward(const nsa_config_t* cfg, const void* q, const void* k, const void* v,
                         const float* gates, const nsa_phi_params_t* phi, float* out,
                         int32_t* sel_idx, float* lse, void* kc_out, void* vc_out, void* workspace,
                         size_t workspace_bytes, void* stream) {
    Shape s;
    NSA_TRY(derive(cfg, s));
    NSA_TRY(supported(s));
    if (cfg->score_map != 0) return NSA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !gates || !out || !sel_idx) return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        (kc_out && !aligned16(kc_out)) || (vc_out && !aligned16(vc_out)))
        return NSA_ERR_INVALID_ARG;
    const FwdWs L = fwd_layout(s);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return NSA_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    const BranchKV kv{k, v, k, v, k, v};
    if (s.DK == 192)
        return forward_impl<192, 128, 16>(s, q, kv, gates, phi, out, sel_idx, lse, kc_out, vc_out, ws, st);
    return forward_impl<64, 64, 4>(s, q, kv, gates, phi, out, sel_idx, lse, kc_out, vc_out, ws, st);
}

nsa_status_t nsa_forward_train(const nsa_config_t* cfg, const void* q, const void* k, const void* v,
                               const float* gates, const nsa_phi_params_t* phi, float* out, int32_t* sel_idx,
                               float* lse, float* o_branch, void* workspace, size_t workspace_bytes,
                               void* stream) {
    Shape s;
    NSA_TRY(derive(cfg, s));
    NSA_TRY(supported(s));
    if (cfg->score_map != 0) return NSA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !gates || !out || !sel_idx || !lse || !o_branch) return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(o_branch))
        return NSA_ERR_INVALID_ARG;
    const FwdWs L = fwd_layout(s);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return NSA_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    const BranchKV kv{k, v, k, v, k, v};
    if (s.DK == 192)
        return forward_impl<192, 128, 16>(s, q, kv, gates, phi, out, sel_idx, lse, nullptr, nullptr, ws, st,
                                          o_branch);
    return forward_impl<64, 64, 4>(s, q, kv, gates, phi, out, sel_idx, lse, nullptr, nullptr, ws, st, o_branch);
}

nsa_status_t nsa_forward_branches(const nsa_config_t* cfg, const void* q, const void* k_cmp,
                                  const void* v_cmp, const void* k_slc, const void* v_slc,
                                  const void* k_win, const void* v_win, const float* gates,
                                  const nsa_phi_params_t* phi, float* out, int32_t* sel_idx, float* lse,
                                  void* kc_out, void* vc_out, void* workspace, size_t workspace_bytes,
                                  void* stream) {
    Shape s;
    NSA_TRY(derive(cfg, s));
    NSA_TRY(supported(s));
    if (cfg->score_map != 0) return NSA_ERR_UNSUPPORTED;
    if (!q || !k_cmp || !v_cmp || !k_slc || !v_slc || !k_win || !v_win || !gates || !out || !sel_idx)
        return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cmp) || !aligned16(v_cmp) || !aligned16(k_slc) || !aligned16(v_slc) ||
        !aligned16(k_win) || !aligned16(v_win) || !aligned16(out) || (kc_out && !aligned16(kc_out)) ||
        (vc_out && !aligned16(vc_out)))
        return NSA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < fwd_branches_total(s) || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return NSA_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    const BranchKV kv{k_cmp, v_cmp, k_slc, v_slc, k_win, v_win};
    if (s.DK == 192)
        return forward_impl<192, 128, 16>(s, q, kv, gates, phi, out, sel_idx, lse, kc_out, vc_out, ws, st);
    return forward_impl<64, 64, 4>(s, q, kv, gates, phi, out, sel_idx, lse, kc_out, vc_out, ws, st);
}

nsa_status_t nsa_select_blocks(const nsa_config_t* cfg, const float* scores, int32_t* sel_idx,
                               void* stream) {
    Shape s;
    NSA_TRY(derive(cfg, s));
    if (!scores || !sel_idx) return NSA_ERR_INVALID_ARG;
    if (s.n > 32 || s.NS > 64 * 32) return NSA_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const long long items = s.B * s.T * s.G;
    const unsigned grid = (unsigned)ceil_div(items, 8);
    if (s.NS <= 32 * 32) {
        NSA_LAUNCH("topn_kernel", st, topn_kernel<32><<<grid, 256, 0, st>>>(scores, items, (int)s.T, (int)s.G,
                                                               (int)s.NS, (int)s.n, (int)s.lp,
                                                               (int)s.fi, (int)s.fl, sel_idx));
    } else {   // longer rows: one CTA per row (the decode step's selection routine)
        NSA_LAUNCH("topn_cta_kernel", st, topn_cta_kernel<<<(unsigned)items, 256, 0, st>>>(scores, (int)s.T, (int)s.G,
                                                               (int)s.NS, (int)s.n, (int)s.lp,
                                                               (int)s.fi, (int)s.fl, sel_idx));
    }
    return last_launch();
}

nsa_status_t nsa_decode(const nsa_config_t* cfg, int32_t num_seqs, const void* q,
                        const void* k_cache, const void* v_cache, const int64_t* kv_offsets,
                        const void* kc_cache, const void* vc_cache, const int64_t* cmp_offsets,
                        const float* gates, float* out, int32_t* sel_idx, float* lse,
                        void* workspace, size_t workspace_bytes, void* stream) {
    Shape s;
    NSA_TRY(derive(cfg, s));
    NSA_TRY(supported(s));
    if (cfg->score_map != 0) return NSA_ERR_UNSUPPORTED;
    if (num_seqs < 0 || num_seqs > cfg->batch) return NSA_ERR_INVALID_ARG;
    if (num_seqs == 0) return NSA_OK;
    if (!q || !k_cache || !v_cache || !kv_offsets || !kc_cache || !vc_cache || !cmp_offsets ||
        !gates || !out || !sel_idx)
        return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(kc_cache) ||
        !aligned16(vc_cache))
        return NSA_ERR_INVALID_ARG;
    const size_t need = decode_ws_bytes(s.B, s.T, s.G, s.l, s.d, s.lp, s.w, s.n, s.DV);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return NSA_ERR_WORKSPACE;
    return decode_impl(s, num_seqs, q, k_cache, v_cache, kv_offsets, kc_cache, vc_cache, cmp_offsets,
                       gates, out, sel_idx, lse, reinterpret_cast<uint8_t*>(workspace),
                       reinterpret_cast<cudaStream_t>(stream));
}

nsa_status_t nsa_decode_rows(const nsa_config_t* cfg, int32_t num_seqs, const void* q,
                             const void* k_cache, const void* v_cache, const int64_t* kv_start,
                             const int64_t* kv_len, const void* kc_cache, const void* vc_cache,
                             const int64_t* cmp_start, const float* gates, float* out, int32_t* sel_idx,
                             float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    Shape s;
    NSA_TRY(derive(cfg, s));
    NSA_TRY(supported(s));
    if (cfg->score_map != 0) return NSA_ERR_UNSUPPORTED;
    if (num_seqs < 0 || num_seqs > cfg->batch) return NSA_ERR_INVALID_ARG;
    if (num_seqs == 0) return NSA_OK;
    if (!q || !k_cache || !v_cache || !kv_start || !kv_len || !kc_cache || !vc_cache || !cmp_start ||
        !gates || !out || !sel_idx)
        return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(kc_cache) ||
        !aligned16(vc_cache))
        return NSA_ERR_INVALID_ARG;
    const size_t need = decode_ws_bytes(s.B, s.T, s.G, s.l, s.d, s.lp, s.w, s.n, s.DV);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return NSA_ERR_WORKSPACE;
    return decode_impl(s, num_seqs, q, k_cache, v_cache, kv_start, kc_cache, vc_cache, cmp_start,
                       gates, out, sel_idx, lse, reinterpret_cast<uint8_t*>(workspace),
                       reinterpret_cast<cudaStream_t>(stream), kv_len);
}

nsa_status_t nsa_decode_append(const nsa_config_t* cfg, int32_t num_seqs, const void* k_new,
                               const void* v_new, void* k_cache, void* v_cache, const int64_t* kv_start,
                               const int64_t* kv_len, void* kc_cache, void* vc_cache,
                               const int64_t* cmp_start, const nsa_phi_params_t* phi, void* stream) {
    Shape s;
    NSA_TRY(derive(cfg, s));
    NSA_TRY(supported(s));
    if (num_seqs < 0) return NSA_ERR_INVALID_ARG;
    if (num_seqs == 0) return NSA_OK;
    if (num_seqs > 65535) return NSA_ERR_UNSUPPORTED;
    if (!k_new || !v_new || !k_cache || !v_cache || !kv_start || !kv_len || !kc_cache || !vc_cache ||
        !cmp_start)
        return NSA_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache))
        return NSA_ERR_INVALID_ARG;
    if (s.phi == NSA_PHI_LINEAR && (!phi || !phi->w_k || !phi->e_k || !phi->w_v || !phi->e_v ||
                                    !aligned16(phi->w_k) || !aligned16(phi->w_v) || !aligned16(phi->e_k) ||
                                    !aligned16(phi->e_v)))
        return NSA_ERR_INVALID_ARG;
    AppendParams p{};
    p.S = num_seqs;
    p.G = (int)s.G;
    p.l = (int)s.l;
    p.d = (int)s.d;
    p.phi = s.phi == NSA_PHI_LINEAR ? 1 : 0;
    p.kv_start = kv_start;
    p.cmp_start = cmp_start;
    p.len = kv_len;
    p.k_new = reinterpret_cast<const __nv_bfloat16*>(k_new);
    p.v_new = reinterpret_cast<const __nv_bfloat16*>(v_new);
    p.k_cache = reinterpret_cast<__nv_bfloat16*>(k_cache);
    p.v_cache = reinterpret_cast<__nv_bfloat16*>(v_cache);
    p.kc_cache = reinterpret_cast<__nv_bfloat16*>(kc_cache);
    p.vc_cache = reinterpret_cast<__nv_bfloat16*>(vc_cache);
    if (p.phi) {
        p.w_k = reinterpret_cast<const __nv_bfloat16*>(phi->w_k);
        p.e_k = reinterpret_cast<const __nv_bfloat16*>(phi->e_k);
        p.w_v = reinterpret_cast<const __nv_bfloat16*>(phi->w_v);
        p.e_v = reinterpret_cast<const __nv_bfloat16*>(phi->e_v);
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const dim3 grid((unsigned)num_seqs, (unsigned)s.G, 2 * kAppendSplit);
    const size_t smem = p.phi ? (size_t)s.l * std::max(s.DK, s.DV) * sizeof(double) : 0;
    if (smem > 48 * 1024) return NSA_ERR_UNSUPPORTED;     // l * d_k <= 6144 for the staged block
    if (s.DK == 192)
        NSA_LAUNCH("decode_append_kernel", st, decode_append_kernel<192, 128><<<grid, 256, smem, st>>>(p));
    else
        NSA_LAUNCH("decode_append_kernel", st, decode_append_kernel<64, 64><<<grid, 256, smem, st>>>(p));
    return last_launch();
}

nsa_status_t nsa_backward(const nsa_config_t* cfg, const void* q, const void* k, const void* v,
                          const float* gates, const nsa_phi_params_t* phi, const void* dout,
                          const int32_t* sel_idx, float* dq, float* dk, float* dv, float* dgates,
                          void* workspace, size_t workspace_bytes, void* stream) {
    Shape s;
    NSA_TRY(derive(cfg, s));
    NSA_TRY(supported(s));
    if (!q || !k || !v || !gates || !dout || !sel_idx || !dq || !dk || !dv || !dgates)
        return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout)) return NSA_ERR_INVALID_ARG;
    const BwdWs L = bwd_layout(s);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return NSA_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    if (s.DK == 192)
        return backward_impl<192, 128>(s, q, k, v, gates, phi, dout, sel_idx, dq, dk, dv, dgates, ws, st);
    return backward_impl<64, 64>(s, q, k, v, gates, phi, dout, sel_idx, dq, dk, dv, dgates, ws, st);
}

nsa_status_t nsa_backward_saved(const nsa_config_t* cfg, const void* q, const void* k, const void* v,
                                const float* gates, const nsa_phi_params_t* phi, const void* dout,
                                const int32_t* sel_idx, const float* lse, const float* o_branch, float* dq,
                                float* dk, float* dv, float* dgates, void* workspace, size_t workspace_bytes,
                                void* stream) {
    Shape s;
    NSA_TRY(derive(cfg, s));
    NSA_TRY(supported(s));
    if (!q || !k || !v || !gates || !dout || !sel_idx || !lse || !o_branch || !dq || !dk || !dv || !dgates)
        return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(o_branch))
        return NSA_ERR_INVALID_ARG;
    const BwdWs L = bwd_layout(s);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return NSA_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    if (s.DK == 192)
        return backward_impl<192, 128>(s, q, k, v, gates, phi, dout, sel_idx, dq, dk, dv, dgates, ws, st, lse,
                                       o_branch);
    return backward_impl<64, 64>(s, q, k, v, gates, phi, dout, sel_idx, dq, dk, dv, dgates, ws, st, lse, o_branch);
}

nsa_status_t nsa_profile_enable(int32_t on) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_on = on != 0;
    return NSA_OK;
}

int32_t nsa_profile_read(int32_t max_kernels, char* names, int32_t* launches, float* total_ms) {
    std::vector<ProfRec> recs;
    {
        std::lock_guard<std::mutex> lk(g_prof_mu);
        recs.swap(g_prof_recs);
    }
    std::vector<std::string> order;
    std::map<std::string, std::pair<int, double>> agg;
    int err = 0;
    for (auto& r : recs) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
            err = 1;
        std::string n(r.name);
        if (!agg.count(n)) order.push_back(n);
        agg[n].first += 1;
        agg[n].second += ms;
    }
    {
        std::lock_guard<std::mutex> lk(g_prof_mu);
        for (auto& r : recs) {
            g_prof_pool.push_back(r.a);
            g_prof_pool.push_back(r.b);
        }
    }
    if (err) return -1;
    int32_t k = 0;
    for (auto& n : order) {
        if (k >= max_kernels) break;
        if (names) {
            std::strncpy(names + 48 * k, n.c_str(), 47);
            names[48 * k + 47] = 0;
        }
        if (launches) launches[k] = agg[n].first;
        if (total_ms) total_ms[k] = (float)agg[n].second;
        ++k;
    }
    return k;
}

nsa_status_t nsa_backward_phi_params(const nsa_config_t* cfg, const void* k, const void* v,
                                     const nsa_phi_params_t* phi, float* dw_k, float* de_k, float* dw_v,
                                     float* de_v, void* workspace, size_t workspace_bytes, void* stream) {
    Shape s;
    NSA_TRY(derive(cfg, s));
    NSA_TRY(supported(s));
    if (s.phi != NSA_PHI_LINEAR) return NSA_ERR_INVALID_ARG;          // mean phi has no parameters
    if (!k || !v || !phi || !phi->w_k || !phi->e_k || !phi->w_v || !phi->e_v || !dw_k || !de_k || !dw_v ||
        !de_v)
        return NSA_ERR_INVALID_ARG;
    if (!aligned16(dw_k) || !aligned16(dw_v)) return NSA_ERR_INVALID_ARG;
    const BwdWs L = bwd_layout(s);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return NSA_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    const int64_t KK = s.l * s.DK, KV = s.l * s.DV;
    if (s.C == 0) {                                      // no compressed block: no gradient
        if (cudaMemsetAsync(dw_k, 0, (size_t)s.DK * KK * 4, st) != cudaSuccess ||
            cudaMemsetAsync(de_k, 0, (size_t)KK * 4, st) != cudaSuccess ||
            cudaMemsetAsync(dw_v, 0, (size_t)s.DV * KV * 4, st) != cudaSuccess ||
            cudaMemsetAsync(de_v, 0, (size_t)KV * 4, st) != cudaSuccess)
            return NSA_ERR_CUDA;
        return NSA_OK;
    }
    const float* dkc = reinterpret_cast<const float*>(ws + L.off_dkc);
    const float* dvc = reinterpret_cast<const float*>(ws + L.off_dvc);
    float* colsum = reinterpret_cast<float*>(ws + L.off_fix);   // scratch: the fix-up list is done
    const int N = (int)(s.B * s.C * s.G);
    auto bf = [](const void* p) { return reinterpret_cast<const __nv_bfloat16*>(p); };
    // column sums in NB row slices (NB + 1 <= N when NB > 1, so the partial sums
    // after the (DK + DV) sums fit in the fix-up scratch of N (DK + DV) floats)
    const int NB = (int)std::min<int64_t>(32, std::max<int64_t>(1, N / 256));
    {
        float* pk = NB > 1 ? colsum + s.DK + s.DV : colsum;
        float* pv = NB > 1 ? pk + (size_t)NB * s.DK : colsum + s.DK;
        NSA_LAUNCH("phi_colsum_kernel", st, phi_colsum_kernel<<<dim3((unsigned)(s.DK / 32), (unsigned)NB), 256, 0, st>>>(dkc, N, (int)s.DK, NB, pk));
        NSA_TRY(last_launch());
        NSA_LAUNCH("phi_colsum_kernel", st, phi_colsum_kernel<<<dim3((unsigned)(s.DV / 32), (unsigned)NB), 256, 0, st>>>(dvc, N, (int)s.DV, NB, pv));
        NSA_TRY(last_launch());
        if (NB > 1) {
            NSA_LAUNCH("phi_colsum_fold", st, phi_colsum_fold<<<(unsigned)ceil_div(s.DK, 64), 64, 0, st>>>(pk, NB, (int)s.DK, colsum));
            NSA_TRY(last_launch());
            NSA_LAUNCH("phi_colsum_fold", st, phi_colsum_fold<<<(unsigned)ceil_div(s.DV, 64), 64, 0, st>>>(pv, NB, (int)s.DV, colsum + s.DK));
            NSA_TRY(last_launch());
        }
    }
    NSA_LAUNCH("phi_de_kernel", st, phi_de_kernel<<<(unsigned)ceil_div(KK, 256), 256, 0, st>>>(bf(phi->w_k), colsum, (int)s.DK, (int)KK, de_k));
    NSA_TRY(last_launch());
    NSA_LAUNCH("phi_de_kernel", st, phi_de_kernel<<<(unsigned)ceil_div(KV, 256), 256, 0, st>>>(bf(phi->w_v), colsum + s.DK, (int)s.DV, (int)KV, de_v));
    NSA_TRY(last_launch());
    if (phi_bwd_tensor_ok(s)) {
        __nv_bfloat16* dyb = reinterpret_cast<__nv_bfloat16*>(ws + L.off_dyb);
        const __nv_bfloat16* dybv = dyb + (size_t)s.B * s.C * s.G * s.DK;
        NSA_TRY(phi_bwd_operands(s, dkc, dvc, dyb, st));
        if (s.DK == 192) {
            NSA_TRY((launch_phi_bwd<192, kPhiDW>(s, dyb, k, nullptr, dw_k, colsum, phi->e_k, st)));
            return launch_phi_bwd<128, kPhiDW>(s, dybv, v, nullptr, dw_v, colsum + s.DK, phi->e_v, st);
        }
        NSA_TRY((launch_phi_bwd<64, kPhiDW>(s, dyb, k, nullptr, dw_k, colsum, phi->e_k, st)));
        return launch_phi_bwd<64, kPhiDW>(s, dybv, v, nullptr, dw_v, colsum + s.DK, phi->e_v, st);
    }
    const int B = (int)s.B, T = (int)s.T, G = (int)s.G, C = (int)s.C, l = (int)s.l, d = (int)s.d;
    if (s.DK == 192) {
        NSA_LAUNCH("phi_dw_kernel", st, phi_dw_kernel<192><<<dim3((unsigned)(KK / 64), 3), 256, 0, st>>>(dkc, bf(k), bf(phi->e_k), B, T, G, C, l, d, dw_k));
        NSA_TRY(last_launch());
        NSA_LAUNCH("phi_dw_kernel", st, phi_dw_kernel<128><<<dim3((unsigned)(KV / 64), 2), 256, 0, st>>>(dvc, bf(v), bf(phi->e_v), B, T, G, C, l, d, dw_v));
    } else {
        NSA_LAUNCH("phi_dw_kernel", st, phi_dw_kernel<64><<<dim3((unsigned)(KK / 64), 1), 256, 0, st>>>(dkc, bf(k), bf(phi->e_k), B, T, G, C, l, d, dw_k));
        NSA_TRY(last_launch());
        NSA_LAUNCH("phi_dw_kernel", st, phi_dw_kernel<64><<<dim3((unsigned)(KV / 64), 1), 256, 0, st>>>(dvc, bf(v), bf(phi->e_v), B, T, G, C, l, d, dw_v));
    }
    return last_launch();
}

nsa_status_t nsa_check_timeout_path(uint64_t limit_ns, void* stream) {
    if (limit_ns == 0 || limit_ns > kWaitLimitNs) return NSA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    NSA_LAUNCH("timeout_selftest_kernel", st, timeout_selftest_kernel<<<1, 32, 0, st>>>(limit_ns));
    return last_launch();
}

nsa_status_t nsa_sync_status(void* stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return NSA_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_nsa_error, sizeof(v)) != cudaSuccess) return NSA_ERR_CUDA;
    if (v) {
        unsigned int z = 0;
        cudaMemcpyToSymbol(g_nsa_error, &z, sizeof(z));
        return (v & 1u) ? NSA_ERR_DEVICE_TIMEOUT : NSA_ERR_INVALID_ARG;
    }
    return NSA_OK;
}

}  // extern "C"

// ===================================================== allocation-free compress
//
// nsa_compress_static: token compression for callers that cannot allocate
// device memory.  Its scratch (the fp64 position-embedding bias and the list
// of elements re-rounded exactly) lives in the fixed array below instead of a
// caller workspace.  The array is a host-side stand-in in host code; its
// device address on the current device is looked up with cudaGetSymbolAddress
// on every call (a host-side query, cheap once the module is loaded), so a
// context that was torn down and re-created never sees a stale address.
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB on every device that loads the library
__device__ __align__(256) uint8_t g_compress_scratch[kStaticScratchBytes];

nsa_status_t static_scratch_ptr(void** out) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_compress_scratch) != cudaSuccess || !p) return NSA_ERR_CUDA;
    *out = p;
    return NSA_OK;
}

}  // namespace

extern "C" nsa_status_t nsa_compress_static(const nsa_config_t* cfg, const void* k, const void* v,
                                            const nsa_phi_params_t* phi, void* kc, void* vc,
                                            void* stream) {
    Shape s;
    NSA_TRY(derive(cfg, s));
    NSA_TRY(supported(s));
    if (!k || !v || !kc || !vc) return NSA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(kc) || !aligned16(vc)) return NSA_ERR_INVALID_ARG;
    const size_t bias_bytes = align256((size_t)(s.DK + s.DV) * 8);
    if (bias_bytes + fix_bytes(s) > kStaticScratchBytes) return NSA_ERR_WORKSPACE;
    void* base = nullptr;
    NSA_TRY(static_scratch_ptr(&base));
    uint8_t* sc = reinterpret_cast<uint8_t*>(base);
    // run_phi clears the fix-up counters at the start of every call
    return run_phi(s, k, v, phi, kc, vc, nullptr, reinterpret_cast<double*>(sc), sc + bias_bytes,
                   reinterpret_cast<cudaStream_t>(stream));
}
