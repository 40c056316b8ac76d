/*
 * hyb_attn.h -- C ABI of the ARL2 hybrid attention layer for NVIDIA B200 (sm_100a).
 *
 * The layer ("Technical summary: Attend Locally, Remember Linearly (ARL2)",
 * gist.science/ar/paper/2605.16579) splits the self-attention of an
 * autoregressive video diffusion transformer into two branches:
 *
 *   §2.1 intra-frame branch   O_intra = softmax(Q K^T * sm_scale) V over the
 *                             tokens of the current frame, bidirectional.
 *   §2.1 inter-frame branch   O_inter = Q' S_{N-1}, with Q' = Q phi_q^T and a
 *                             fixed-size per-head fp32 state S (d_k x d_v).
 *   §2.1 state update         S_N = alpha S_{N-1} + K'^T diag(beta) (V' - K' S_{N-1})
 *                             (printed garbled on the page; this is the only
 *                             shape-consistent reading), K' = rownorm(K phi_k^T),
 *                             V' = V phi_v^T, beta_t = sigmoid(beta_logit_t),
 *                             alpha = mean_t sigmoid(gate_logit_t) (one forget
 *                             gate per head and frame, §4 "headwise gating").
 *   §2.2 frame-level access   every token of a frame reads the same pre-update
 *                             S_{N-1}; the state is written after the reads.
 *   §2.2 clean-pass updates   denoising passes (clean_pass = 0) read S and never
 *                             write it; the final clean pass (clean_pass = 1)
 *                             writes it once.
 *
 * Readings where the pages are silent (all are choices of this library):
 *   - output      out = O_intra + O_inter, rounded once to the I/O dtype
 *                 (the pages do not say how the branches combine;
 *                 hyb_attn_forward_mixed weights the two branches);
 *   - 1x1 maps    x'[o] = sum_i phi[o][i] x[i], i.e. X' = X phi^T; no bias,
 *                 no nonlinearity; the same q, k, v feed both branches;
 *   - K' only     is L2-normalised, as k / sqrt(sum k^2 + l2_eps);
 *   - sm_scale    defaults to 1/sqrt(d_k);
 *   - alpha       is the mean of the per-token sigmoids, not the sigmoid of
 *                 the mean logit.
 *
 * Layouts (row-major, contiguous, every pointer 16-byte aligned):
 *   q, k, v, out          [B][T][H][d]     dtype (bf16 or fp32)
 *   phi_q, phi_k, phi_v   [H][d][d]        dtype, phi[h][o][i]
 *   gate_logits,
 *   beta_logits           [B][H][T]        fp32 (read only when clean_pass)
 *   state                 [B][H][d_k][d_v] fp32, read always, written only
 *                                           when clean_pass
 *   out_intra, out_inter  [B][T][H][d]     fp32 (debug entry point)
 *
 * Supported shapes: d_k == d_v == 128 with bf16 I/O (tensor-core path), and
 * d_k == d_v == 32 with fp32 I/O (fp32 SIMT path).  Any T >= 1, B >= 1, H >= 1
 * with B*H*T*d below 2^31 elements.  Other combinations return
 * HYB_ERR_UNSUPPORTED.
 *
 * Ownership: the caller owns every buffer, including the persistent state and
 * the workspace; the library never allocates, frees or synchronises inside
 * hyb_attn_forward*.  The state persists across calls: the caller passes
 * S_{N-1} for frame N and zero-fills it for S_0.  The caller zero-fills the
 * workspace once after allocating it (its first 256 bytes hold the device
 * status flags).  Calls are asynchronous on the given stream; argument errors
 * are reported before anything is launched.  `stream` is a cudaStream_t
 * (NULL = legacy default stream).  Calls sharing one workspace must be ordered
 * on one stream.  No C++ exception crosses this interface.
 */
#ifndef HYB_ATTN_H
#define HYB_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HYB_OK = 0,
    HYB_WARN_NONFINITE = 1,   /* device flag: a state update produced inf/NaN      */
    HYB_ERR_INVALID = -1,     /* null pointer, non-positive size, bad flag          */
    HYB_ERR_UNSUPPORTED = -2, /* (dtype, d) combination not built                   */
    HYB_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned                   */
    HYB_ERR_WORKSPACE = -4,   /* workspace null or smaller than hyb_attn_workspace_bytes */
    HYB_ERR_CUDA = -5,        /* a CUDA runtime/driver call or a launch failed      */
    HYB_ERR_TIMEOUT = -6      /* device flag: a bounded device-side wait gave up    */
} hyb_status;

typedef enum { HYB_BF16 = 0, HYB_FP32 = 1 } hyb_dtype;

typedef struct {
    int B, H, T, d_k, d_v;
    int dtype;        /* hyb_dtype: dtype of q, k, v, phi_*, out                 */
    float sm_scale;   /* softmax scale; <= 0 selects 1/sqrt(d_k)                 */
    float l2_eps;     /* key-normalisation epsilon (>= 0); 1e-6 is the default   */
} hyb_attn_desc;

/* Bytes of device workspace one call with this descriptor needs (0 if the
 * descriptor is invalid or unsupported).  It is linear in B*H and does not
 * depend on the frame count. */
size_t hyb_attn_workspace_bytes(const hyb_attn_desc* desc);

/* One pass of the layer over one frame (ARL2 summary §2.1, §2.2).
 * clean_pass = 0: query-only denoising pass; reads state, never writes it;
 *                 gate_logits / beta_logits may be NULL.
 * clean_pass = 1: also applies the gated delta update to state in place,
 *                 after every read of S_{N-1} for this frame's output.
 * Writes out = O_intra + O_inter.  Returns HYB_OK once the work is enqueued. */
hyb_status hyb_attn_forward(const hyb_attn_desc* desc,
                            const void* q, const void* k, const void* v,
                            const void* phi_q, const void* phi_k, const void* phi_v,
                            const float* gate_logits, const float* beta_logits,
                            float* state, int clean_pass, void* out,
                            void* workspace, size_t workspace_bytes, void* stream);

/* hyb_attn_forward_next -- the same pass as hyb_attn_forward (same arguments,
 * bit-identical outputs and state), for one call per pass in a stream of passes
 * (autoregressive use: the next frame's inputs exist only after this frame).
 * The inter-frame read needs W = phi_q^T S_{N-1} (ARL2 summary §2.1); a clean
 * pass's delta update already holds S_N, so here it also writes the next
 * frame's W (the prep kernel's operands and instruction sequence), and the next
 * call continues from it: no prep kernel, and its attention kernel starts
 * while this pass's update still runs.  A call continues the chain when the
 * previous pass on this workspace was a hyb_attn_forward_next call with the same
 * descriptor, state, phi_q and stream; any other call (or a pass of any other
 * entry point on this workspace or state) starts a new chain, which runs the
 * prep kernel first, exactly as hyb_attn_forward.
 * Caller's contract while a chain runs: nothing but these calls writes the
 * state, phi_q or the workspace.  A caller that resets or restores the state
 * starts the next chain with a hyb_attn_forward call (or any other pass on
 * that workspace), which ends the old chain; the library cannot see a write
 * the caller makes itself.  The chained update releases the next one through
 * flag words in the workspace (a bounded device wait: HYB_ERR_TIMEOUT after
 * 2 s).  The chain record is kept on the host for up to 16 workspaces; not
 * thread-safe.  The fp32 path keeps no chain (each call is hyb_attn_forward). */
hyb_status hyb_attn_forward_next(const hyb_attn_desc* desc,
                                 const void* q, const void* k, const void* v,
                                 const void* phi_q, const void* phi_k, const void* phi_v,
                                 const float* gate_logits, const float* beta_logits,
                                 float* state, int clean_pass, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* Same pass, also writing the two branches separately in fp32 (for parity
 * checks); out may be NULL, out_intra and out_inter may not. */
hyb_status hyb_attn_forward_branches(const hyb_attn_desc* desc,
                                     const void* q, const void* k, const void* v,
                                     const void* phi_q, const void* phi_k, const void* phi_v,
                                     const float* gate_logits, const float* beta_logits,
                                     float* state, int clean_pass, void* out,
                                     float* out_intra, float* out_inter,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* hyb_attn_forward_frames -- n_frames consecutive frames of one stream, each a
 * clean pass (hyb_attn_forward with clean_pass = 1, frame after frame), in one
 * call.  Frame N's inter-frame read needs W_N = phi_q^T S_{N-1} only at the
 * end of its attention kernel, and frame N's state update never waits for
 * frame N's attention, so the call runs the short sequential chain (W_N, then
 * S_N, frame after frame) on one internal stream and the attention kernels on
 * two others, frame after frame in turn, each attention kernel waiting only for
 * its own W_N: the attention kernels of consecutive frames share the SMs, and
 * consecutive state updates overlap (the next walks its key tiles while the
 * current one reduces and writes the state; flag words in the workspace order
 * their accesses to the state, with a bounded device wait).  The
 * results are bit-identical to the loop: the same kernels with the same
 * arithmetic; only their scheduling differs (for the fp32 path the call is the
 * loop).  The internal streams (the chain's at the highest priority) and events
 * are created on the first call on a device and kept; the call forks from and
 * joins back to `stream`, so work enqueued on `stream` afterwards sees every
 * output and the final state.  Not thread-safe.
 *   q, k, v, out: [n_frames][B][T][H][d]; gate_logits, beta_logits:
 *   [n_frames][B][H][T] fp32 (B*H*T a multiple of 4, so every frame's gate
 *   pointer stays 16-byte aligned; HYB_ERR_ALIGN otherwise); state: S_{-1} on
 *   entry (the state before the first frame), the state after the last frame
 *   on return.  workspace: hyb_attn_frames_workspace_bytes(desc, n_frames)
 *   bytes (it grows with n_frames: one W per frame), zero-filled once.
 * HYB_ERR_INVALID if n_frames is outside [1, 4096]; otherwise the errors of
 * hyb_attn_forward, checked for every frame before anything is enqueued. */
size_t hyb_attn_frames_workspace_bytes(const hyb_attn_desc* desc, int n_frames);
hyb_status hyb_attn_forward_frames(const hyb_attn_desc* desc, int n_frames,
                                   const void* q, const void* k, const void* v,
                                   const void* phi_q, const void* phi_k, const void* phi_v,
                                   const float* gate_logits, const float* beta_logits,
                                   float* state, void* out,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* hyb_attn_forward_mixed -- the same pass with a per-(batch, head) weighting of
 * the two branches: out = a * O_intra + c * O_inter, with (a, c) = mix[b][h]
 * ([B][H][2] fp32, device memory, 16-byte aligned).  It carries the branch
 * combinations of the adjacent methods as scalars the caller supplies:
 * LinVideo ("LinVideo: A Post-Training Framework towards O(n) Attention in
 * Efficient Video Generation", §2(b) selective transfer) mixes
 * r * softmax + (1 - r) * linear, i.e. (a, c) = (r, 1 - r); SALAD ("SALAD:
 * Achieve High-Sparsity Attention via Efficient Linear Attention Tuning for
 * Video Diffusion Transformer", §2 static-dynamic scaling) scales the linear
 * branch by a learned static gain g, (1, g), or by a sigmoid-bounded dynamic
 * factor s = sigmoid(z) computed by the caller, (1, s).  (1, 1) is
 * hyb_attn_forward.  The state update is unchanged.  c is applied to
 * W = phi_q^T S_{N-1} before the read (exact: Q (c W) = c O_inter) and a in the
 * output epilogue.  HYB_ERR_INVALID if mix or out is NULL; otherwise the
 * arguments and errors of hyb_attn_forward. */
hyb_status hyb_attn_forward_mixed(const hyb_attn_desc* desc,
                                  const void* q, const void* k, const void* v,
                                  const void* phi_q, const void* phi_k, const void* phi_v,
                                  const float* gate_logits, const float* beta_logits,
                                  float* state, int clean_pass, const float* mix, void* out,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* hyb_attn_forward_noalloc -- the same pass as hyb_attn_forward for callers
 * that cannot allocate device memory: code running where cudaMalloc is
 * forbidden or unavailable (inside a CUDA graph being captured with a strict
 * capture mode, inside an allocator or memory-pool callback, in a real-time
 * or pre-sized serving loop whose memory budget is fixed up front).  No
 * counterpart in the paper: this is an interface convenience only.
 *
 * Instead of a caller workspace it uses one scratch array of
 * HYB_NOALLOC_SCRATCH_BYTES held by the library on every GPU that loads it,
 * for as long as the process runs.  The call allocates nothing (no cudaMalloc,
 * cudaFree or allocating library routine); the caller still passes every input
 * and output.  A descriptor whose hyb_attn_workspace_bytes() exceeds
 * HYB_NOALLOC_SCRATCH_BYTES is rejected with HYB_ERR_WORKSPACE before any
 * launch.  The first call on a device looks up the scratch array's device
 * address (cudaGetSymbolAddress) with that device current; make that first
 * call before any stream capture.  All calls on a device share the one array
 * and it keeps the last call's contents: calls that can overlap on the GPU
 * (different streams, concurrent threads) race on it and must be serialised by
 * the caller.  Device status flags of these calls are cleared at the start of
 * each call; hyb_attn_noalloc_device_status reports those of the last call. */
#define HYB_NOALLOC_SCRATCH_BYTES (32u << 20)
hyb_status hyb_attn_forward_noalloc(const hyb_attn_desc* desc,
                                    const void* q, const void* k, const void* v,
                                    const void* phi_q, const void* phi_k, const void* phi_v,
                                    const float* gate_logits, const float* beta_logits,
                                    float* state, int clean_pass, void* out, void* stream);

/* hyb_attn_noalloc_device_status -- synchronises `stream`, then reads and
 * clears the device status flags of the last hyb_attn_forward_noalloc call on
 * the current device (in the library's scratch array), with the meaning of
 * hyb_attn_get_device_status.  HYB_OK if no such call was made on this device.
 * Allocates nothing. */
hyb_status hyb_attn_noalloc_device_status(void* stream);

/* hyb_attn_forward_token_level -- the token-level access variant of a pass
 * (ARL2 summary §4, ablations: token-level against frame-level access to the
 * memory).  The pages give it no formulas; the reading taken: on a clean pass
 * the tokens of the frame update the state one after another by the
 * frame-level rule applied to a single token, with a per-token forget gate,
 *     S_t = alpha_t S_{t-1} + beta_t k'_t (v'_t - k'_t^T S_{t-1}),
 *     alpha_t = sigmoid(gate_logit_t), beta_t = sigmoid(beta_logit_t),
 * and token t reads the state before its own update, O_inter[t] = q'_t S_{t-1}
 * (causal within the frame).  The residual is taken against the undecayed
 * state, as in the frame-level rule, so a one-token frame gives the same update
 * under both accesses (this is not the decayed residual of "Gated Delta
 * Networks").  out = O_intra + O_inter, rounded once; state holds S_{N-1} on
 * entry and the state after the frame's last token on return.  A query-only
 * pass (clean_pass = 0) is exactly hyb_attn_forward's.  Computed in chunks of
 * 64 tokens in fp32 with only relative decays exp(Lambda_a - Lambda_b) <= 1.
 * Same arguments, layouts, alignment and errors as hyb_attn_forward, except the
 * workspace: at least hyb_attn_token_level_workspace_bytes(desc) bytes
 * (HYB_ERR_WORKSPACE otherwise), zero-filled once like hyb_attn_forward's. */
size_t hyb_attn_token_level_workspace_bytes(const hyb_attn_desc* desc);
hyb_status hyb_attn_forward_token_level(const hyb_attn_desc* desc,
                                        const void* q, const void* k, const void* v,
                                        const void* phi_q, const void* phi_k, const void* phi_v,
                                        const float* gate_logits, const float* beta_logits,
                                        float* state, int clean_pass, void* out,
                                        void* workspace, size_t workspace_bytes, void* stream);

/* hyb_tra_forward -- the hybrid layer with Token Radius Attention on its
 * intra-frame branch ("Technical summary: Token Radius Attention",
 * gist.science/ar/paper/2608.02504, §2): each query attends only to the key
 * blocks near it on the frame's patch grid, with a radius set by its attention
 * entropy.  warmup = 1: the dense pass of hyb_attn_forward (same outputs, same
 * state update) that also writes every query's attention entropy
 * H = -sum_j p_j ln p_j (nats) to `entropy` ([B][H][T] fp32, 16-byte aligned)
 * and then builds the block mask from them in the workspace.  warmup = 0: the
 * intra-frame attention runs block-sparse with the mask the last warm-up pass on
 * this workspace built (the page computes the entropies once and reuses them
 * across the later denoising steps; with no mask built yet the pass is dense;
 * `entropy` is not read).  The mask: the entropies give each query a budget
 * k = clamp(tau exp(H), 1, T) keys and a disk radius r = sqrt(k / pi) patches
 * (the page's temporal decay exp(-gamma delta) is 1 on the current frame, the
 * only one this branch attends to); a query votes for a key block when some key
 * of it lies within r (Euclidean distance on patch coordinates); a key block is
 * kept for a query block with at least votes_min votes, and always for itself;
 * the intra-frame attention of each query then runs over the kept blocks of its
 * query block (the block-sparse result).  The inter-frame read and the state
 * update are those of hyb_attn_forward.  Blocks are runs of 128 tokens of the
 * frame, which must be in tile-major order: tiles of tile_h x tile_w patches
 * taken row-major over the grid_h x grid_w grid (grid_h * grid_w == T), patches
 * row-major inside a tile, edge tiles cut by the grid; the caller orders q, k, v
 * (and reads out) that way.  bf16 with d = 128 only (HYB_ERR_UNSUPPORTED
 * otherwise) and T <= 28288 (221 key blocks: the mask kernel keeps every key
 * block's bounding box and row runs in shared memory; HYB_ERR_UNSUPPORTED
 * beyond).  workspace: hyb_tra_workspace_bytes(desc), zero-filled once.
 * HYB_ERR_INVALID for bad params (grid sides >= 32768, tau <= 0 or not finite,
 * votes_min < 1) or warmup outside {0, 1}; otherwise hyb_attn_forward's errors. */
typedef struct {
    int grid_h, grid_w;   /* the frame's patch grid (grid_h * grid_w == T) */
    int tile_h, tile_w;   /* tile-major order */
    float tau;            /* budget scale: k = tau exp(H) keys */
    int votes_min;        /* votes that keep a key block (>= 1) */
} hyb_tra_params;
size_t hyb_tra_workspace_bytes(const hyb_attn_desc* desc);
hyb_status hyb_tra_forward(const hyb_attn_desc* desc, const hyb_tra_params* params, int warmup,
                           const void* q, const void* k, const void* v,
                           const void* phi_q, const void* phi_k, const void* phi_v,
                           const float* gate_logits, const float* beta_logits,
                           float* state, int clean_pass, void* out, float* entropy,
                           void* workspace, size_t workspace_bytes, void* stream);

/* hyb_kvcache_attn_forward -- the softmax baseline the hybrid layer replaces
 * (ARL2 summary §1, problem statement: softmax self-attention whose key/value
 * cache grows with every generated chunk; §4, the memory and wall-clock
 * comparison against it).  One call per frame: the frame's k and v
 * ([B][T][H][128] bf16) are copied into rows [cached_tokens, cached_tokens+T)
 * of each batch's cache, then every query of the frame attends, with softmax
 * scale desc->sm_scale (<= 0: 1/sqrt(128)), over all cached_tokens + T keys:
 *     out = softmax(q k_cache^T * scale) v_cache,
 * bidirectional within the frame and over every earlier frame, no inter-frame
 * read and no state.  The caller tracks cached_tokens (0 for the first frame;
 * add T after each call).
 *   k_cache, v_cache: [B][cache_tokens][H][128] bf16, caller-owned; rows
 *       >= cached_tokens + T are never read.
 *   out: [B][T][H][128] bf16.  workspace: at least 256 bytes, zero-filled once
 *       (device status flags, read by hyb_attn_get_device_status).
 * desc: B, H, T, d_k = d_v = 128, dtype HYB_BF16 (else HYB_ERR_UNSUPPORTED);
 * l2_eps is ignored.  HYB_ERR_INVALID if cached_tokens < 0 or
 * cached_tokens + T > cache_tokens; HYB_ERR_ALIGN if a pointer is not 16-byte
 * aligned; HYB_ERR_WORKSPACE if the workspace is missing or too small.
 * Asynchronous on `stream`, like hyb_attn_forward. */
hyb_status hyb_kvcache_attn_forward(const hyb_attn_desc* desc, const void* q, const void* k, const void* v,
                                    void* k_cache, void* v_cache, int cache_tokens, int cached_tokens,
                                    void* out, void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then reads and clears the device status flags kept
 * in `workspace`: HYB_ERR_CUDA if a kernel found its launch environment
 * unusable (e.g. a misaligned shared-memory window) and did nothing,
 * else HYB_ERR_TIMEOUT if a bounded device wait gave up,
 * else HYB_WARN_NONFINITE if a state update produced inf/NaN since the last
 * read, else HYB_OK (or HYB_ERR_CUDA if the synchronisation failed). */
hyb_status hyb_attn_get_device_status(const void* workspace, void* stream);

/* ---- fault test (tests only) --------------------------------------------------
 * Process-wide and off by default; affects calls made after it, on any device.
 * wait_limit_us > 0 replaces the 2 s limit of the attention kernel's bounded
 * device waits (mbarrier waits) by that many microseconds (at most 10 s);
 * 0 restores 2 s.  skip_v_loads = 1 makes the attention kernel's value-tile
 * producer issue no loads at all, so the first wait for a value tile expires:
 * the kernel then sets the TIMEOUT flag that hyb_attn_get_device_status reports
 * as HYB_ERR_TIMEOUT, stores no output, waits for the products it has issued,
 * frees its tensor memory and returns, leaving the device usable.  No copy is
 * in flight when the wait expires.  The delta update is not affected.
 * HYB_ERR_INVALID for skip_v_loads outside {0, 1} or a limit above 10 s.
 * Not thread-safe; set it back to (0, 0) after the test. */
hyb_status hyb_attn_set_fault_test(int skip_v_loads, unsigned wait_limit_us);

/* ---- optional kernel timing (benchmarks) ------------------------------------
 * Process-wide and off by default.  hyb_attn_timing_begin(n) creates 2n CUDA
 * events on the current device; until hyb_attn_timing_end, every kernel that
 * hyb_attn_forward* or hyb_kvcache_attn_forward (as "intra_frame_attention")
 * launches is bracketed by two of them on the call's stream
 * (launches beyond n are counted as dropped).  Do not leave timing on while a
 * stream is being captured into a CUDA graph.  hyb_attn_timing_end waits for
 * the recorded events, sums each kernel's launch count and event time into
 * *out, destroys the events and turns timing off.  Not thread-safe. */
#define HYB_NUM_KERNELS 7
typedef struct {
    int launches[HYB_NUM_KERNELS];     /* indexed as hyb_attn_kernel_name() */
    double total_ms[HYB_NUM_KERNELS];
    int dropped;
} hyb_attn_timing;

hyb_status hyb_attn_timing_begin(int max_launches);
hyb_status hyb_attn_timing_end(hyb_attn_timing* out);
/* "prep", "intra_frame_attention", "delta_update" (bf16: the whole update; fp32:
 * its token-split reduction), "delta_update_apply" (fp32 only), and the three
 * kernels of a token-level clean pass: "token_chunk_prep", "token_chain",
 * "token_reads"; NULL if out of range */
const char* hyb_attn_kernel_name(int kernel);

/* Static string naming a status code. */
const char* hyb_attn_status_string(hyb_status status);

#ifdef __cplusplus
}
#endif

#endif /* HYB_ATTN_H */
