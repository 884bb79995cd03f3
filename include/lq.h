/*
 * liblq: windowed INT8 recurrent-state decode for gated delta-rule linear
 * attention on NVIDIA B200 (sm_100a).  C ABI.
 *
 * Sources.  Each declaration below names the passage that defines what it
 * computes:
 *   [abs]  the paper page "LeapQuant: Efficient Linear Attention with
 *          Accurate Recurrent State Quantization" (mlsanity.com), section
 *          "Abstract (arXiv)";
 *   [news] the bedrocknews.com article on arXiv 2609.38166v1, its paragraph
 *          on the mechanism (FP32 inference as the baseline, naive per-token
 *          quantization as the failing alternative, outlier rows and columns
 *          kept in FP16/FP32).
 * The pages define no programming interface.  Calls that only manage memory,
 * handles, errors or checkpoints say "Source: none" and have no counterpart
 * in the pages.
 *
 * The method (LeapQuant, arXiv 2609.38166, [abs]): each (sequence, head)
 * pair of a Gated DeltaNet (GDN) or Kimi Delta Attention (KDA) layer keeps a
 * d_v x d_k recurrent state S.  The state
 * is stored as 8-bit codes and is quantized only once per window of W tokens;
 * within a window, outputs come from the fixed low-bit state together with
 * high-precision buffered updates.  The largest outlier rows and columns of
 * the state are kept in FP32 as Compensator Tokens that share the update path
 * of real tokens, and the remaining residual is smoothed before it is
 * quantized.
 *
 * Recurrences (the published GDN rule; for KDA the per-key-channel gate
 * multiplies the key side):
 *   GDN: S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *   KDA: S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *   o_t = S_t q_t.
 * The gate is passed as g_t = log(alpha_t).  q is used as given (no 1/sqrt(d)
 * scaling).
 *
 * Stored window-start state per (sequence, head): codes Q (int8, d_v x d_k),
 * row scales sigma (FP32, d_v), column smoothing factors s (FP32, d_k) and
 * compensators C = sum_c v_c k_c^T (FP32 rank-1 pairs: a row compensator is
 * (e_i, S[i,:]), a column compensator is (S[:,j], e_j)).  Decoded state:
 * S~_ij = sigma_i Q_ij s_j + C_ij.
 *
 * Conventions for every call:
 *  - Memory.  The caller owns all device memory.  It allocates one workspace
 *    of lq_workspace_bytes() bytes (256-byte aligned) and passes device
 *    pointers; liblq allocates nothing on the device.  A handle owns only host
 *    metadata.  Inputs are read during the call's kernels and not retained.
 *  - Streams.  `stream` is a cudaStream_t (NULL = legacy default stream).  All
 *    device work is enqueued on it, asynchronously; no call synchronizes except
 *    lq_device_status() and lq_state_export().
 *  - Overlapped launches.  The windowed decode kernel is launched as a
 *    programmatic dependent of the kernel before it in the stream: its CTAs
 *    set up while that kernel finishes, and read the step's inputs and the
 *    window buffer only after it has completed.  When the handle's previous
 *    call that enqueued device work was also a decode, a CTA fetches its
 *    first INT8 code tile before that point too; the workspace's codes must
 *    therefore not be written by any means but this library's calls.  A
 *    caller that writes the encoded state itself (a checkpoint restore) calls
 *    lq_state_resume() afterwards: the decode after it fetches nothing early.
 *  - Errors.  Every call returns an lq_status.  Errors found on the host are
 *    returned at once and leave the state untouched; the text of the last one
 *    on the calling thread is lq_last_error_string().  Errors found on the
 *    device (a gate sum out of the safe range, a bounded wait that expired)
 *    are recorded in the workspace's error word and reported by
 *    lq_device_status().  No kernel traps or asserts.  A state whose error
 *    word is set is to be prefilled again before further use: the launch that
 *    recorded the error may have left it partly updated.
 *  - Tracing.  Every call that enqueues device work opens an NVTX range named
 *    after the call, so timeline tools group its kernels under it.
 *  - Window phase.  By default all sequences of a handle share one window
 *    phase: the handle counts buffered tokens (lq_window_fill) on the host.
 *    A ragged handle (cfg.ragged = 1, windowed mode) keeps one count per
 *    (sequence, head) on the device instead, so that sequences can skip
 *    steps, join and leave independently (continuous batching); see
 *    lq_decode_step_active(), lq_window_flush(), lq_window_flush_pending()
 *    and lq_prefill_sequences().
 *  - Threads.  A handle must not be used by two threads at once; different
 *    handles may be used from different host threads concurrently.
 */
#ifndef LQ_H
#define LQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LQ_API __attribute__((visibility("default")))
#else
#define LQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lq_status {
    LQ_OK = 0,
    LQ_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad handle, bad field   */
    LQ_ERR_UNSUPPORTED = 2,  /* valid request outside the compiled kernels        */
    LQ_ERR_WORKSPACE = 3,    /* workspace too small or misaligned                 */
    LQ_ERR_WINDOW_FULL = 4,  /* decode with W tokens buffered: flush first        */
    LQ_ERR_RANGE = 5,        /* device: gate sum outside the safe range           */
    LQ_ERR_CUDA = 6,         /* a CUDA runtime call failed (text has the reason)  */
    LQ_ERR_DEVICE = 7,       /* device: another error recorded in the error word  */
    LQ_ERR_STATE = 8         /* call out of order (e.g. decode before prefill)    */
} lq_status;

enum { LQ_GATE_SCALAR = 0 /* GDN */, LQ_GATE_CHANNEL = 1 /* KDA */ };
enum {
    LQ_MODE_WINDOW = 0,  /* windowed INT8 state (the method)                 */
    LQ_MODE_NAIVE = 1,   /* per-token requantized INT8 state (comparator)     */
    LQ_MODE_FP32 = 2     /* FP32 state, plain recurrence (comparator)         */
};
enum { LQ_SELECT_L2 = 0, LQ_SELECT_MAXABS = 1 };
enum { LQ_DTYPE_F32 = 0, LQ_DTYPE_BF16 = 1 };

/* Device error codes in the workspace error word (lq_layout.err, int32[0]).
 * LQ_DEVERR_BOUNDS: a computed index outside its region, whose access was
 * skipped.  The bounds-checked build of the library (liblq_checked.so) checks
 * the indices it derives from workspace contents; every build checks the unit
 * tickets, which are out of range when a launch that ended on a device error
 * left a ticket counter set (prefill clears it).  lq_device_status() reports
 * it as LQ_ERR_DEVICE. */
enum { LQ_DEVERR_NONE = 0, LQ_DEVERR_RANGE = 1, LQ_DEVERR_TIMEOUT = 2, LQ_DEVERR_WINDOW_FULL = 3,
       LQ_DEVERR_BOUNDS = 4 };

typedef struct lq_config {
    int32_t batch;        /* sequences, >= 1                                     */
    int32_t heads;        /* heads per sequence, >= 1                            */
    int32_t d_k;          /* key channels: 64 or 128                             */
    int32_t d_v;          /* value channels: equal to d_k                        */
    int32_t window;       /* W, tokens per window, 1..4096 (windowed mode)       */
    int32_t n_comp_rows;  /* compensator rows, 0..8 (windowed mode)              */
    int32_t n_comp_cols;  /* compensator columns, 0..8 (windowed mode)           */
    int32_t gate;         /* LQ_GATE_SCALAR or LQ_GATE_CHANNEL                   */
    int32_t mode;         /* LQ_MODE_*                                           */
    int32_t smooth;       /* 1: column smoothing before quantization (windowed)  */
    int32_t select;       /* compensator ranking: LQ_SELECT_L2 or _MAXABS        */
    int32_t in_dtype;     /* dtype of q, k, v: LQ_DTYPE_BF16 or LQ_DTYPE_F32     */
    int32_t ragged;       /* 1: per-(sequence, head) window phases on the device
                             (windowed mode only); 0: one shared phase         */
} lq_config;

/*
 * Byte offsets of the regions of a workspace (each 256-byte aligned), for
 * callers that inspect or checkpoint the state.  N = batch * heads, units in
 * (sequence, head) order; absent regions have offset LQ_ABSENT.
 */
#define LQ_ABSENT ((size_t)-1)
typedef struct lq_layout {
    size_t total_bytes;
    size_t err;           /* int32[64]: [0] LQ_DEVERR_*, [1] unit, [2] detail;
                             [32..33], [34..35] unit-ticket counters of the
                             windowed decode and the window flush: zero
                             between launches (prefill clears them)          */
    size_t codes;         /* int8  [N][d_v][d_k]                 window, naive    */
    size_t row_scale;     /* f32   [N][d_v]       sigma          window, naive    */
    size_t col_smooth;    /* f32   [N][d_k]       s              window           */
    size_t comp_index;    /* int32 [N][comp_index_stride]: rows then columns      */
    size_t comp_row_vec;  /* f32   [N][n_comp_rows][d_k]  k of row compensators   */
    size_t comp_col_vec;  /* f32   [N][n_comp_cols][d_v]  v of column comps       */
    size_t gate_sum;      /* f64   [N][1 (GDN) or d_k (KDA)]: sum of g this window*/
    size_t buf_delta;     /* f32   [N][window][d_v]  buffered delta_j             */
    size_t buf_key;       /* GDN: in_dtype [N][window][d_k] k_j;
                             KDA: f32 [N][window][d_k] k_j * exp(-G_j)            */
    size_t buf_gate;      /* f32   [N][window_pad] exp(-G_j) (GDN only)           */
    size_t state_f32;     /* f32   [N][d_v][d_k]                  FP32 mode        */
    int32_t comp_index_stride;  /* n_comp_rows + n_comp_cols rounded up to 4      */
    int32_t window_pad;         /* window rounded up to 4                          */
    size_t fill;          /* int32 [N] tokens buffered per unit (0..W)   ragged     */
} lq_layout;

typedef struct lq_state_s *lq_handle;

/* Bytes of device workspace a config needs; 0 if the config is invalid.
 * Source: none (memory sizing). */
LQ_API size_t lq_workspace_bytes(const lq_config *cfg);

/* Fill *out with the workspace layout of a valid config.  The layout is
 * internal and may change between versions: read the state through
 * lq_state_export(); use the layout only to checkpoint whole workspaces.
 * Source: none (memory layout). */
LQ_API lq_status lq_workspace_layout(const lq_config *cfg, lq_layout *out);

/*
 * Create a handle over a caller-owned workspace (d_workspace: device pointer,
 * 256-byte aligned, `bytes` >= lq_workspace_bytes(cfg)).  Host-only: touches
 * no device memory.  The state is undefined until lq_prefill_state().
 * Source: [abs] (one recurrent state per (sequence, head) of a GDN or KDA
 * layer, held in 8 bits); the handle itself has no counterpart.
 */
LQ_API lq_status lq_state_create(const lq_config *cfg, void *d_workspace, size_t bytes, lq_handle *out);

/*
 * Ingest a prefilled FP32 state and start the first window (the state is
 * quantized once per window, at its end; the end of the prefill is the start
 * of the first window).
 * d_S0: device FP32 [batch][heads][d_v][d_k], or NULL for an all-zero state.
 *   windowed: the codec (compensator extraction, smoothing, per-row INT8);
 *   naive:    per-row INT8 without compensators or smoothing;
 *   FP32:     a copy.
 * Clears the error word, the gate sums and the window buffer.
 * Source: [abs] (the state is quantized once per window, at its end, with
 * the largest outliers kept as Compensator Tokens and the residual smoothed
 * before quantization); [news] for the naive and FP32 comparators.
 */
LQ_API lq_status lq_prefill_state(lq_handle h, const float *d_S0, void *stream);

/*
 * One decode token for every (sequence, head): the output is formed from the
 * INT8 window-start state plus the FP32 buffered updates of the window.
 * Device inputs, unit-major [batch][heads][.], 16-byte aligned:
 *   d_q, d_k: [.][d_k], d_v: [.][d_v] in cfg.in_dtype;
 *   d_g: log alpha, f32 [.] (GDN) or [.][d_k] (KDA);  d_beta: f32 [.];
 * output d_o: f32 [.][d_v], o_t = S_t q_t.
 * Windowed mode reads the INT8 window-start state once, adds the buffered
 * corrections, appends (delta_t, key_t, G_t) to the buffer and writes no
 * state; it returns LQ_ERR_WINDOW_FULL when W tokens are already buffered.
 * Naive mode updates and requantizes the INT8 state; FP32 mode updates it.
 * On a ragged handle this is lq_decode_step_active() with every sequence active.
 * Source: [abs] (outputs from the fixed low-bit state plus high-precision
 * buffered updates; Compensator Tokens on the update path of real tokens);
 * [news] (the FP32-state baseline and naive per-token quantization).
 */
LQ_API lq_status lq_decode_step(lq_handle h, const void *d_q, const void *d_k, const void *d_v,
                         const float *d_g, const float *d_beta, float *d_o, void *stream);

/*
 * Ragged handles: one decode token for every active sequence.  d_active:
 * device uint8 [batch], nonzero = this sequence takes a token this step; NULL =
 * all.  Inputs and outputs as lq_decode_step(); the rows of inactive sequences
 * are not read, their outputs not written and their windows not advanced.  A
 * unit whose window already holds W tokens is skipped and LQ_DEVERR_WINDOW_FULL
 * recorded (lq_device_status() returns LQ_ERR_WINDOW_FULL): call
 * lq_window_flush() after every step.  LQ_ERR_STATE on a shared-phase handle.
 * The beta and g entries of inactive sequences may be read (a prefetch) but
 * never affect any result; their q, k, v rows are not read.
 * Source: [abs] (the windowed scheme, applied to each sequence over its own
 * tokens; the pages do not discuss sequences that join or skip steps).
 */
LQ_API lq_status lq_decode_step_active(lq_handle h, const void *d_q, const void *d_k, const void *d_v,
                                       const float *d_g, const float *d_beta, const uint8_t *d_active,
                                       float *d_o, void *stream);

/*
 * End the window (windowed mode; a no-op returning LQ_OK otherwise): rebuild
 * the state in FP32 from the window-start state and the buffered updates,
 * take the new Compensator Tokens (largest rows, then columns), smooth the
 * residual and requantize it to per-row INT8; empty the buffer.  Allowed with
 * any number of buffered tokens, including none.  On a ragged handle only the
 * units whose window holds W tokens are flushed (the others are untouched).
 * Cost on a ragged handle: until an active mask or lq_prefill_sequences() is
 * used (counting from lq_prefill_state() or lq_window_flush_pending()), every
 * unit is in the same phase, which the handle follows on the host: the call
 * launches nothing when no window is full and otherwise flushes like a
 * shared-phase handle.  Once phases differ, a launch reads every unit's count
 * and re-encodes only the due units.
 * Source: [abs] (quantized a single time, at the end of the window; largest
 * outliers kept as high-precision Compensator Tokens; residual smoothed
 * before quantization); [news] (the outliers are whole rows and columns).
 */
LQ_API lq_status lq_window_flush(lq_handle h, void *stream);

/*
 * Ragged handles: flush every unit holding at least one buffered token (for
 * example before a sequence leaves).  Shared-phase handles: lq_window_flush().
 * Source: [abs], as lq_window_flush() (a window that ends early).
 */
LQ_API lq_status lq_window_flush_pending(lq_handle h, void *stream);

/*
 * Ragged handles: start new sequences in some batch slots.  The sequences with
 * d_mask[b] != 0 (device uint8 [batch]) are encoded from d_S0 (device FP32
 * [batch][heads][d_v][d_k], only their rows read; NULL = all-zero state) and
 * their windows emptied; the other sequences are untouched.  Requires a prior
 * lq_prefill_state(); LQ_ERR_STATE on a shared-phase handle.
 * Source: [abs], as lq_prefill_state().
 */
LQ_API lq_status lq_prefill_sequences(lq_handle h, const float *d_S0, const uint8_t *d_mask, void *stream);

/*
 * Prefill from prompt tokens: run the FP32 recurrence of the gated delta rule
 * over n_tokens prompt tokens of every sequence, starting from d_S0 (device
 * FP32 [batch][heads][d_v][d_k]; NULL = all-zero state), and make the state
 * after the last token the window-start state, exactly as lq_prefill_state()
 * would from that FP32 state: encoded (windowed and naive modes) or stored
 * (FP32 mode).  The prompt runs at full precision; the codec of LeapQuant
 * ("LeapQuant: Efficient Linear Attention with Accurate Recurrent State
 * Quantization", section "Abstract (arXiv)") applies once, at its end.
 * Inputs are token-major, each token laid out as for lq_decode_step():
 *   d_q, d_k, d_v: in_dtype [n_tokens][batch][heads][d]  (16-byte aligned);
 *   d_g: f32 [n_tokens][batch][heads] (GDN) or [..][d_k] (KDA, 16-byte aligned);
 *   d_beta: f32 [n_tokens][batch][heads].
 * d_o: f32 [n_tokens][batch][heads][d_v], o_t = S_t q_t for every prompt
 * token, or NULL to skip the outputs.  n_tokens = 0 is lq_prefill_state().
 * Afterwards every window is empty (ragged handles: every count is 0 and the
 * phases are aligned).  The caller keeps ownership of every buffer; nothing is
 * retained after the call.  Errors: LQ_ERR_INVALID_ARG for a NULL input with
 * n_tokens > 0, a negative n_tokens or a misaligned pointer.
 * Source: [abs] (the codec once, at the end of the prompt; the pages do not
 * say how a prompt is ingested, so the prompt itself runs in FP32).
 */
LQ_API lq_status lq_prefill_tokens(lq_handle h, const float *d_S0, const void *d_q, const void *d_k,
                                   const void *d_v, const float *d_g, const float *d_beta, int32_t n_tokens,
                                   float *d_o, void *stream);

/*
 * Ragged handles: start new sequences in some batch slots from their prompts,
 * as lq_prefill_sequences() does from a state.  The sequences with
 * d_mask[b] != 0 (device uint8 [batch]) run the FP32 recurrence from d_S0
 * (their rows; NULL = zero state) over their first d_lengths[b] prompt tokens
 * (device int32 [batch], clamped to 0..max_tokens; NULL = max_tokens for
 * all), and the state after them is encoded as their window-start state, with
 * their windows emptied.  Prompt inputs are laid out as for
 * lq_prefill_tokens() over max_tokens tokens; only the rows of masked
 * sequences and of their own tokens are read, and only those outputs are
 * written (d_o may be NULL).  Other sequences are untouched.  Requires a prior
 * lq_prefill_state(); LQ_ERR_STATE on a shared-phase handle; LQ_ERR_INVALID_ARG
 * for a NULL mask, a negative max_tokens, a NULL input with max_tokens > 0 or a
 * misaligned pointer.
 * Source: [abs], as lq_prefill_tokens().
 */
LQ_API lq_status lq_prefill_sequences_tokens(lq_handle h, const float *d_S0, const void *d_q, const void *d_k,
                                             const void *d_v, const float *d_g, const float *d_beta,
                                             int32_t max_tokens, const int32_t *d_lengths, const uint8_t *d_mask,
                                             float *d_o, void *stream);

/*
 * Resume from a checkpoint.  A handle's whole state is its workspace plus, for
 * a shared-phase handle, the host count lq_window_fill().  To checkpoint: call
 * lq_device_status() (it synchronizes the stream), then copy the workspace's
 * lq_workspace_bytes() bytes and note lq_window_fill().  To resume: create a
 * handle with the same lq_config over a workspace holding those bytes (the
 * copy may sit at another address or on another device), then call this with
 * the noted count.  n_buf: tokens buffered in the shared window, 0..W
 * (windowed mode), 0 in the other modes; a ragged handle takes its counts
 * from the workspace and ignores n_buf (pass 0).  No device work; the next
 * decode, flush or prefill continues exactly where the checkpoint stood, and
 * the next decode reads the codes only after the kernel before it in its
 * stream has completed.
 * Errors: LQ_ERR_INVALID_ARG for a bad handle or an n_buf out of range.
 * Source: none (checkpointing).
 */
LQ_API lq_status lq_state_resume(lq_handle h, int32_t n_buf);

/*
 * Destination buffers of lq_state_export(), N = batch * heads units in
 * (sequence, head) order, each region packed with no padding.  Every pointer
 * may be NULL (that region is not copied) or point to device memory or to
 * host memory (pinned or pageable); the caller owns them.  A non-NULL pointer
 * for a region the handle's mode does not keep is an error.
 */
typedef struct lq_export {
    int8_t *codes;          /* int8  [N][d_v][d_k]   Q             windowed, naive */
    float *row_scale;       /* f32   [N][d_v]        sigma         windowed, naive */
    float *col_smooth;      /* f32   [N][d_k]        s             windowed        */
    int32_t *comp_index;    /* int32 [N][n_comp_rows + n_comp_cols]: rows, columns */
    float *comp_row_vec;    /* f32   [N][n_comp_rows][d_k]  k of row compensators  */
    float *comp_col_vec;    /* f32   [N][n_comp_cols][d_v]  v of column comps      */
    float *buf_delta;       /* f32   [N][window][d_v]  buffered delta_j            */
    void *buf_key;          /* [N][window][d_k]: GDN in_dtype k_j; KDA f32
                               k_j * exp(-G_j)                                     */
    float *buf_gate;        /* f32   [N][window]  exp(-G_j) of entry j (GDN)       */
    double *gate_sum;       /* f64   [N][1 (GDN) or d_k (KDA)]: G of the window    */
    int32_t *fill;          /* int32 [N] tokens buffered per unit, 0..W (windowed
                               mode, shared or ragged phases)                      */
    float *state_f32;       /* f32   [N][d_v][d_k]                 FP32 mode       */
} lq_export;

/*
 * Copy the current state into caller buffers (see lq_export): the stored
 * window-start state (codes, row scales, smoothing factors, Compensator
 * Tokens), the window's buffered entries and their count, or the FP32 state.
 * Buffer entries past a unit's count are copied but hold no meaning.
 * Enqueues the copies on `stream`, then synchronizes it (like
 * lq_device_status()) and reads the device error word.  Returns LQ_OK; the
 * device status (LQ_ERR_RANGE, LQ_ERR_WINDOW_FULL or LQ_ERR_DEVICE, text in
 * lq_last_error_string()) when the error word is set, in which case the
 * copied state may be inconsistent; LQ_ERR_INVALID_ARG for a bad handle, a
 * NULL dst or a pointer for an absent region (nothing is copied);
 * LQ_ERR_STATE before lq_prefill_state(); LQ_ERR_CUDA when a copy fails.
 * Source: [abs] (the fixed low-bit state: 8-bit codes plus high-precision
 * buffered updates and Compensator Tokens); [news] for the FP32 state.
 */
LQ_API lq_status lq_state_export(lq_handle h, const lq_export *dst, void *stream);

/* Tokens buffered in the current window (0..W); -1 for a bad or ragged handle
 * (a ragged handle's counts are on the device: lq_state_export() reads them).
 * Source: [abs] (the window of W tokens). */
LQ_API int32_t lq_window_fill(lq_handle h);

/*
 * Synchronize `stream` and read the device error word: LQ_OK, LQ_ERR_RANGE,
 * LQ_ERR_WINDOW_FULL or LQ_ERR_DEVICE (detail in lq_last_error_string()).
 * Source: none (error reporting).
 */
LQ_API lq_status lq_device_status(lq_handle h, void *stream);

/* Release the handle (host metadata only; the workspace stays the caller's).
 * Source: none. */
LQ_API lq_status lq_state_destroy(lq_handle h);

/* Text of the last error on the calling thread ("" if none).  Source: none. */
LQ_API const char *lq_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* LQ_H */
