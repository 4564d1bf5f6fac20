/*
 * nsa.h -- C ABI of libnsa, a B200 (sm_100a) implementation of the Native
 * Sparse Attention (NSA) per-layer attention operator.
 *
 * What the operator computes (page "硬件对齐+原生训练！DeepSeek NSA打造高效稀疏
 * Attention", section 二 NSA核心工作; explainer "DeepseekNativelySparseAttention",
 * sections on compressed / selected / sliding-window attention and the gated
 * fusion):  for every query token t and query head h of a causal GQA context
 *
 *     out[t,h] = g_cmp[t,h] * Attn(q[t,h], K~cmp, V~cmp)
 *              + g_slc[t,h] * Attn(q[t,h], K[selected blocks], V[...])
 *              + g_win[t,h] * Attn(q[t,h], K[t-w+1 .. t], V[...])
 *
 * with Attn(q, K, V) = softmax(scale * q K^T) V over the keys that branch
 * remaps (token compression, top-n block selection, sliding window):
 *   - compressed keys/values: K~[i] = phi(k[i*d .. i*d+l-1]) for blocks of
 *     length l at stride d (phi = mean-pool, or a linear map of the flattened
 *     block plus an intra-block position embedding), rounded to bf16; block i
 *     is visible to t once complete (i*d + l - 1 <= t);
 *   - selected blocks: selection blocks of l' tokens; importance
 *     p'[t,g,j] = sum over the heads h of group g of sum_i w(i,j) p_cmp[t,h,i],
 *     where p_cmp is the compressed branch's softmax and w(i,j) counts the
 *     stride-d segments compressed block i shares with selection block j;
 *     the first `forced_initial` blocks and the `forced_local` blocks ending
 *     at floor(t/l') are always kept, the remaining n - forced are the
 *     highest-scoring other candidates (ties to the lower index); when at most
 *     n candidate blocks exist all are taken;
 *   - window: the last w tokens up to and including t.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers to contiguous row-major arrays
 *     owned by the caller; libnsa never allocates, frees or synchronises
 *     device memory during a call.  Scratch memory is the caller-provided
 *     workspace (size from nsa_workspace_size), 256-byte aligned.
 *   - bf16 tensors (q, k, v, phi parameters, caches, dout) are bfloat16;
 *     gates, out, lse and gradients are fp32; indices int32; offsets int64.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  The returned status covers argument validation and
 *     kernel launch.  A device-side failure (a bounded wait that expired) is
 *     reported by nsa_sync_status().
 *   - Invalid arguments return NSA_ERR_INVALID_ARG and launch nothing.
 *     Valid but unimplemented shapes return NSA_ERR_UNSUPPORTED.
 */
#ifndef NSA_H_
#define NSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NSA_OK = 0,
    NSA_ERR_INVALID_ARG = 1,   /* null pointer, inconsistent sizes, bad hyperparameters */
    NSA_ERR_UNSUPPORTED = 2,   /* valid, but no kernel instantiated for these sizes */
    NSA_ERR_WORKSPACE = 3,     /* workspace missing, misaligned or too small */
    NSA_ERR_CUDA = 4,          /* a CUDA runtime/driver call or launch failed */
    NSA_ERR_DEVICE_TIMEOUT = 5 /* a kernel's bounded wait expired (see nsa_sync_status) */
} nsa_status_t;

typedef enum { NSA_PHI_MEAN = 0, NSA_PHI_LINEAR = 1 } nsa_phi_t;

typedef enum {
    NSA_MODE_FORWARD = 0,
    NSA_MODE_DECODE = 1,
    NSA_MODE_BACKWARD = 2,
    NSA_MODE_FORWARD_BRANCHES = 3 /* nsa_forward_branches */
} nsa_mode_t;

/* Operator configuration.  Token compression: block length l = cmp_block,
 * stride d = cmp_stride.  Selection: block length l' = sel_block, n =
 * sel_count blocks of which forced_initial + forced_local are always kept.
 * Window: w = window tokens.  Requirements (validated): d divides l and l';
 * l <= l'; n >= forced_initial + forced_local; num_q_heads a multiple of
 * num_kv_groups.  Implemented sizes: (d_k, d_v) in {(64,64), (192,128)},
 * heads per group in {4, 16}, l/d in {1, 2}, l'/d in {1, 2, 4}, score_map 0.
 * For nsa_decode, `batch` is the number of sequences and `seqlen` the largest
 * context length (they size the workspace). */
typedef struct {
    int32_t batch, seqlen, num_q_heads, num_kv_groups, d_k, d_v;
    int32_t cmp_block, cmp_stride, sel_block, sel_count, forced_initial, forced_local, window;
    int32_t phi;       /* nsa_phi_t */
    int32_t score_map; /* 0: overlap-weighted mapping of compressed to selection blocks */
    float scale;       /* softmax scale; 0 selects 1/sqrt(d_k) */
} nsa_config_t;

/* Linear phi parameters (bf16, device): w_k [d_k, l*d_k], e_k [l, d_k],
 * w_v [d_v, l*d_v], e_v [l, d_v].  The flattened block is position-major:
 * x[j*d_k + c] = k[i*d + j][c] + e_k[j][c], K~[i] = w_k x.  Unused (may be
 * NULL) for NSA_PHI_MEAN. */
typedef struct {
    const void* w_k;
    const void* e_k;
    const void* w_v;
    const void* e_v;
} nsa_phi_params_t;

/* Bytes of device workspace an entry point needs for this configuration. */
size_t nsa_workspace_size(const nsa_config_t* cfg, int32_t mode);

/* Number of compressed blocks over a context of `len` tokens:
 * floor((len - l)/d) + 1, or 0 when len < l (token compression section). */
int64_t nsa_num_cmp_blocks(const nsa_config_t* cfg, int64_t len);

/* Token compression alone (page 2, 令牌压缩; explainer 2.2-2.3).
 * k [B,T,G,d_k], v [B,T,G,d_v] -> kc [B,C,G,d_k], vc [B,C,G,d_v] (bf16,
 * round-to-nearest-even), C = nsa_num_cmp_blocks(cfg, T).  Needs the FORWARD
 * workspace. */
nsa_status_t nsa_compress(const nsa_config_t* cfg, const void* k, const void* v,
                          const nsa_phi_params_t* phi, void* kc, void* vc, void* workspace,
                          size_t workspace_bytes, void* stream);

/* Token compression without any device allocation.  No counterpart in the
 * paper: this entry point exists for callers that cannot call cudaMalloc or
 * hand over a workspace -- code running inside CUDA graph capture, plugins
 * hosted by a framework that owns all device memory, or a serving loop that
 * must not allocate per step while it appends compressed blocks to its
 * cache.  It computes exactly what nsa_compress computes (same kernels, same
 * outputs), with its scratch in a fixed 16 MiB device array compiled into
 * the library (held by every GPU that loads it, until process exit):
 *   - sizes: 8*(d_k + d_v) rounded up to 256, plus 256 + 4*B*C*G*(d_k + d_v)
 *     bytes must fit in 16 MiB, otherwise NSA_ERR_WORKSPACE is returned and
 *     nothing is launched (e.g. B=1, G=4, d_k+d_v=320 allows up to about
 *     T=52k tokens);
 *   - every call looks up the array's device address on the current device
 *     (a host-side query); the first call on a device may load the library's
 *     device code there, so make that first call before any stream capture;
 *   - all calls share the array: two calls whose kernels overlap on the GPU
 *     (different streams, or different host threads on one device) race;
 *     serialise them.  Each call clears the counters it needs.
 * Arguments as in nsa_compress, without the workspace. */
nsa_status_t nsa_compress_static(const nsa_config_t* cfg, const void* k, const void* v,
                                 const nsa_phi_params_t* phi, void* kc, void* vc, void* stream);

/* Prefill forward (page 2, sections 整体框架 / 算法设计 / 最终输出计算).
 * In:  q [B,T,H,d_k], k [B,T,G,d_k], v [B,T,G,d_v] bf16; gates [B,T,H,3] fp32
 *      in the order (compressed, selected, window), the sigmoid outputs.
 * Out: out [B,T,H,d_v] fp32; sel_idx [B,T,G,n] int32 (ascending, -1 padded);
 *      lse [B,T,H,3] fp32 natural-log log-sum-exp of each branch's scaled
 *      logits (-inf where a branch sees no key) or NULL;
 *      kc_out [B,C,G,d_k] / vc_out [B,C,G,d_v] bf16 compressed keys/values or
 *      NULL.  sel_idx is required. */
nsa_status_t nsa_forward(const nsa_config_t* cfg, const void* q, const void* k, const void* v,
                         const float* gates, const nsa_phi_params_t* phi, float* out,
                         int32_t* sel_idx, float* lse, void* kc_out, void* vc_out,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Prefill forward with independent keys and values per branch (page 2, 滑动窗口:
 * the three branches are given their own keys and values, so that the local
 * window cannot take over what compression and selection should learn).
 * The compressed branch compresses k_cmp [B,T,G,d_k] / v_cmp [B,T,G,d_v]
 * (phi as in nsa_compress; its probabilities also drive the selection), the
 * selected branch attends the chosen blocks of k_slc / v_slc, the window the
 * last w tokens of k_win / v_win; all bf16, same shapes as k / v of
 * nsa_forward.  Everything else (q, gates, phi, outputs, errors) as in
 * nsa_forward; with the same tensor passed for all three branches the results
 * equal nsa_forward's bit for bit.  Needs the NSA_MODE_FORWARD_BRANCHES
 * workspace (one transposed copy of v_win more than NSA_MODE_FORWARD; the
 * score table sits at the same offset, see nsa_forward_score_table). */
nsa_status_t nsa_forward_branches(const nsa_config_t* cfg, const void* q, const void* k_cmp,
                                  const void* v_cmp, const void* k_slc, const void* v_slc,
                                  const void* k_win, const void* v_win, const float* gates,
                                  const nsa_phi_params_t* phi, float* out, int32_t* sel_idx, float* lse,
                                  void* kc_out, void* vc_out, void* workspace, size_t workspace_bytes,
                                  void* stream);

/* Where nsa_forward leaves the group importance scores (page 2, 重要性分数计算:
 * the compressed branch's probabilities mapped onto selection blocks by the
 * overlap weights and summed over the heads of a GQA group), the table the
 * top-n step reads.  Returns the byte offset of the table inside the FORWARD
 * workspace, or -1 for an invalid cfg; *row_stride (if not NULL) receives NSp,
 * the padded number of selection blocks per row.  After an nsa_forward call
 * with this cfg has completed, p'[b,t,g,j] is the fp32 at
 * workspace + offset + 4*(((b*T + t)*G + g)*NSp + j) for every block
 * j <= floor(t / sel_block) of a row that sees at least one compressed block
 * (t >= cmp_block - 1); other entries are unspecified.  The table stays valid
 * until the workspace is reused.  No device work, no CUDA call. */
int64_t nsa_forward_score_table(const nsa_config_t* cfg, int64_t* row_stride);

/* Batched decode step (page 2, 效率分析 解码速度): one query per sequence at
 * position t = L_s - 1 over caches that already hold the current token.
 * q [S,H,d_k] bf16; k_cache [sumL,G,d_k], v_cache [sumL,G,d_v] bf16 with
 * sequence s in rows [kv_offsets[s], kv_offsets[s+1]); kc_cache [sumC,G,d_k],
 * vc_cache [sumC,G,d_v] bf16 with sequence s in rows [cmp_offsets[s],
 * cmp_offsets[s+1]), which must number nsa_num_cmp_blocks(cfg, L_s);
 * offsets are int64 device arrays of S+1 entries; gates [S,H,3] fp32.
 * Out: out [S,H,d_v] fp32, sel_idx [S,G,n] int32, lse [S,H,3] fp32 or NULL.
 * At most 2048 sequences per call (NSA_ERR_UNSUPPORTED beyond).
 * num_seqs must not exceed cfg->batch and no L_s may exceed cfg->seqlen (the
 * workspace was sized from them): a longer context is skipped on the device
 * and reported as NSA_ERR_INVALID_ARG by nsa_sync_status().  A compressed
 * cache of the wrong length is not detected: that sequence's result is
 * undefined. */
nsa_status_t nsa_decode(const nsa_config_t* cfg, int32_t num_seqs, const void* q,
                        const void* k_cache, const void* v_cache, const int64_t* kv_offsets,
                        const void* kc_cache, const void* vc_cache, const int64_t* cmp_offsets,
                        const float* gates, float* out, int32_t* sel_idx, float* lse,
                        void* workspace, size_t workspace_bytes, void* stream);

/* Backward with the block selection held fixed (pages: natively trainable
 * design; training-speed paragraph of 效率分析).  In: the forward inputs, the
 * upstream gradient dout [B,T,H,d_v] bf16 and sel_idx [B,T,G,n] (normally the
 * forward's).  Out (fp32, overwritten): dq [B,T,H,d_k], dk [B,T,G,d_k],
 * dv [B,T,G,d_v] (through all three branches and, for the compressed branch,
 * through phi), dgates [B,T,H,3] = <dout, o_branch>.  The per-branch softmax
 * statistics are recomputed (each branch once more forward under sel_idx), so
 * any valid selection may be passed.  No gradient flows into the importance
 * scores, the phi parameters or the gate MLP.  The BACKWARD workspace holds,
 * besides the compressed keys and their gradients, one fp32 [B,T,H,d_v] branch
 * output (about 1.1 GB at B=2, T=16384, H=64). */
nsa_status_t nsa_backward(const nsa_config_t* cfg, const void* q, const void* k, const void* v,
                          const float* gates, const nsa_phi_params_t* phi, const void* dout,
                          const int32_t* sel_idx, float* dq, float* dk, float* dv, float* dgates,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Training forward (pages: natively trainable design; 最终输出计算 for the
 * gated sum): exactly nsa_forward (same kernels, same out, sel_idx and lse,
 * bit for bit), and in addition each branch's own output before its gate,
 * which is what the backward's per-branch statistics are made of.
 * Out: out, sel_idx as nsa_forward; lse [B,T,H,3] fp32 (required);
 *      o_branch [3,B,T,H,d_v] fp32 (required, 16-byte aligned): o_cmp, o_slc,
 *      o_win in that order, each normalised by its own softmax, so that
 *      out = sum_c gates[..., c] * o_branch[c] up to rounding.
 * Same FORWARD workspace as nsa_forward; the compressed keys are not
 * returned (the backward recomputes them). */
nsa_status_t nsa_forward_train(const nsa_config_t* cfg, const void* q, const void* k, const void* v,
                               const float* gates, const nsa_phi_params_t* phi, float* out, int32_t* sel_idx,
                               float* lse, float* o_branch, void* workspace, size_t workspace_bytes,
                               void* stream);

/* Backward from the training forward's saved statistics: as nsa_backward, but
 * the per-branch outputs and LSEs are read from `o_branch` and `lse` as
 * nsa_forward_train wrote them for the same q, k, v, phi and sel_idx,
 * instead of being recomputed by three more forward passes (the usual
 * attention-training split: the forward keeps what the softmax backward
 * needs).  Results equal nsa_backward's up to the order of floating-point
 * additions.  Passing statistics that belong to other inputs gives wrong
 * gradients; nothing checks them.  BACKWARD workspace, as nsa_backward. */
nsa_status_t nsa_backward_saved(const nsa_config_t* cfg, const void* q, const void* k, const void* v,
                                const float* gates, const nsa_phi_params_t* phi, const void* dout,
                                const int32_t* sel_idx, const float* lse, const float* o_branch, float* dq,
                                float* dk, float* dv, float* dgates, void* workspace, size_t workspace_bytes,
                                void* stream);

/* Batched decode step over caches with spare capacity per sequence: as
 * nsa_decode, but sequence s holds kv_len[s] tokens in rows [kv_start[s],
 * kv_start[s] + kv_len[s]) of k_cache/v_cache and nsa_num_cmp_blocks(cfg,
 * kv_len[s]) compressed blocks from row cmp_start[s] of kc_cache/vc_cache
 * (kv_start, kv_len, cmp_start: int64 device arrays of S entries).  With
 * nsa_decode_append this serves a generation loop without repacking the
 * caches.  Same limits, workspace and errors as nsa_decode. */
nsa_status_t nsa_decode_rows(const nsa_config_t* cfg, int32_t num_seqs, const void* q,
                             const void* k_cache, const void* v_cache, const int64_t* kv_start,
                             const int64_t* kv_len, const void* kc_cache, const void* vc_cache,
                             const int64_t* cmp_start, const float* gates, float* out, int32_t* sel_idx,
                             float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* Decode-step cache maintenance (page 2, 令牌压缩: block i covers tokens
 * [i*d, i*d + l); 效率分析 解码速度: the decode step reads the compressed cache).
 * Appends one token per sequence and compresses the block it completes.
 * In:  k_new [S,G,d_k], v_new [S,G,d_v] bf16: the token at position kv_len[s]
 *      of sequence s; kv_start, kv_len, cmp_start as for nsa_decode_rows
 *      (lengths BEFORE the append); phi parameters for NSA_PHI_LINEAR.
 * Out: row kv_start[s] + kv_len[s] of k_cache/v_cache; and when the new length
 *      L = kv_len[s] + 1 satisfies L >= l and (L - l) % d == 0, row
 *      cmp_start[s] + (L - l)/d of kc_cache/vc_cache = phi of tokens
 *      [L - l, L), correctly rounded to bf16 (each output one fp64 sum).
 * The caller owns the capacity (the rows written must exist) and advances
 * kv_len itself after the call.  Needs no workspace; S <= 65535; caches, new
 * rows and phi parameters 16-byte aligned (NSA_ERR_INVALID_ARG otherwise). */
nsa_status_t nsa_decode_append(const nsa_config_t* cfg, int32_t num_seqs, const void* k_new,
                               const void* v_new, void* k_cache, void* v_cache, const int64_t* kv_start,
                               const int64_t* kv_len, void* kc_cache, void* vc_cache,
                               const int64_t* cmp_start, const nsa_phi_params_t* phi, void* stream);

/* Top-n block selection alone (page 2, Top-n 块选择; its hyperparameter
 * paragraph fixes 1 initial and 2 local blocks as always selected), the step
 * nsa_forward takes between the compressed and the selected branch.
 * In:  scores [B,T,G,NS] fp32, NS = ceil(T / sel_block): importance score of
 *      selection block j for query token t and GQA group g.  Only blocks
 *      0 .. floor(t / sel_block) of row t are read.  Scores are >= 0; a
 *      negative or NaN score is never selected (the slot stays -1).
 * Out: sel_idx [B,T,G,n] int32, ascending, -1 padded: all blocks when at most
 *      n exist; otherwise blocks 0 .. forced_initial-1, the forced_local
 *      blocks ending at floor(t / sel_block), and the n - forced_initial -
 *      forced_local highest scores among the remaining blocks, ties to the
 *      lower block index (decided on the fp32 values).
 * Needs no workspace.  NSA_ERR_UNSUPPORTED when sel_count > 32 or NS > 2048;
 * the head dimensions and compression sizes of cfg are not used. */
nsa_status_t nsa_select_blocks(const nsa_config_t* cfg, const float* scores, int32_t* sel_idx,
                               void* stream);

/* Gradients of the linear phi's parameters (page 2, 令牌压缩: a learnable map
 * with intra-block position encoding, K~[i] = w_k vec(k_blk + e_k), likewise
 * V~).  Reads the compressed-key gradients dK~/dV~ that the preceding
 * nsa_backward call with the same cfg left in `workspace` (same stream, the
 * workspace untouched in between) and k, v, phi as passed to it.
 * Out (fp32, caller-owned): dw_k [d_k, l*d_k], de_k [l, d_k], dw_v [d_v, l*d_v],
 * de_v [l, d_v]:  dW[o, x] = sum over (b, block i, g) of dK~[o] * x[x] with
 * x = vec(k_blk + e_k);  dE[j, c] = sum over o of w[o, j*d + c] * sum dK~[o].
 * NSA_ERR_INVALID_ARG for the mean phi (no parameters) or missing tensors. */
nsa_status_t nsa_backward_phi_params(const nsa_config_t* cfg, const void* k, const void* v,
                                     const nsa_phi_params_t* phi, float* dw_k, float* de_k, float* dw_v,
                                     float* de_v, void* workspace, size_t workspace_bytes, void* stream);

/* Failure-detection self-test: launches one kernel whose single waiting thread
 * waits, through the same bounded wait every libnsa kernel uses, on an
 * mbarrier on which nothing ever arrives.  After limit_ns nanoseconds of device
 * time (1 .. 2e9) the wait gives up, records its site in the device error word
 * and the kernel returns normally: the next nsa_sync_status() on that stream
 * reports NSA_ERR_DEVICE_TIMEOUT and clears the word, and the CUDA context
 * stays usable.  No fault, trap or hang is involved.  NSA_ERR_INVALID_ARG for a
 * limit outside that range.  Not part of the pages' operator: it lets a caller
 * (and the test suite) check that an expired wait is reported. */
nsa_status_t nsa_check_timeout_path(uint64_t limit_ns, void* stream);

/* Synchronise `stream`, then read and clear the device error word of the
 * current device.  Returns NSA_ERR_DEVICE_TIMEOUT if a kernel's bounded wait
 * expired since the last call, NSA_ERR_CUDA if synchronisation failed. */
nsa_status_t nsa_sync_status(void* stream);

/* Per-kernel timing, for diagnostics and benchmarking.  While enabled (on =
 * 1), every kernel launch made by the entry points is bracketed by two CUDA
 * events recorded on the call's stream (events are created by the library,
 * no device memory is allocated).  nsa_profile_read() waits for the recorded
 * events and fills, per kernel name (at most max_kernels, 48-byte
 * NUL-terminated names), the number of launches and the total device time in
 * ms since the previous read, then clears the records; it returns the number
 * of names written, or -1 on a CUDA error.  Not thread-safe against
 * concurrent entry-point calls from other host threads. */
nsa_status_t nsa_profile_enable(int32_t on);
int32_t nsa_profile_read(int32_t max_kernels, char* names, int32_t* launches, float* total_ms);

/* Static description of a status code. */
const char* nsa_status_string(nsa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* NSA_H_ */
