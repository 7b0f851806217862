/*
 * gdn.h -- C ABI of libgdn.so: the gated delta-rule linear-attention operator
 * on NVIDIA B200 (sm_100a).
 *
 * The operator (state stored as M = S^T, one d_k x d_v matrix per sequence and
 * head):
 *     M_t = (I - beta_t k_t k_t^T) Diag(a_t) M_{t-1} + beta_t k_t v_t^T
 *     o_t = M_t^T q_t
 * with a_t = exp(g_t), either one scalar per token and head (Gated DeltaNet)
 * or one value per key dimension (the per-dimension gate).  Sources: the delta
 * rule as an online gradient step ("OSDN: Improving Delta Rule with Provable
 * Online Preconditioning in Linear Attention", sec. 1) and its scalar- and
 * per-dimension-gated forms ("Moonshot AI's New Attention Architecture: Key
 * Innovations Explained", sec. 2 Core Operator).  With S = M^T this is
 * S_t = S_{t-1} Diag(a_t)(I - beta_t k_t k_t^T) + beta_t v_t k_t^T, the form in
 * which an exact write (beta = 1, |k| = 1) gives S_t k_t = v_t.
 *
 * Conventions shared by every entry point:
 *   - Ownership: the caller owns every buffer (inputs, outputs, workspace).
 *     The library never allocates or frees memory.
 *   - Execution: every call only enqueues work on `stream` and returns; it
 *     never synchronizes (gdn_read_device_status excepted).  Outputs are valid
 *     once the stream has reached the enqueued work.
 *   - Errors: argument errors are detected on the host before anything is
 *     enqueued and return a status; nothing is launched and no output is
 *     touched.  A failed launch returns GDN_ERR_CUDA.  Nothing throws.
 *   - Pointers are device pointers (or managed memory) and must be 16-byte
 *     aligned; tensors are dense and row-major in the layouts given below.
 *   - q and k are used as given: no L2 normalisation and no 1/sqrt(d) scale.
 *   - beta and g have the same element type as q, k, v; states are fp32.
 */
#ifndef GDN_H
#define GDN_H

#include <stddef.h>

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ABI-identical to cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st* gdn_stream_t;

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,  /* null or misaligned pointer, negative size, bad overlap */
    GDN_ERR_UNSUPPORTED = 2,  /* valid request outside the built shapes / dtypes */
    GDN_ERR_WORKSPACE = 3,    /* workspace smaller than gdn_chunk_fwd_workspace_min_bytes */
    GDN_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed */
    GDN_ERR_TIMEOUT = 5       /* a kernel gave up a bounded wait (reported by
                                 gdn_read_device_status) */
} gdn_status;

typedef enum { GDN_BF16 = 0, GDN_F32 = 1 } gdn_dtype;

typedef enum {
    GDN_GATE_NONE = 0,     /* a_t = 1 (DeltaNet)                     */
    GDN_GATE_SCALAR = 1,   /* g: [.., H]      one log-decay per head */
    GDN_GATE_PER_DIM = 2   /* g: [.., H, Dk]  one log-decay per key dimension */
} gdn_gate;

/*
 * gdn_chunk_fwd -- chunkwise forward over a whole sequence batch.
 *
 * Computes o_t for every token and (optionally) the final state, splitting
 * each sequence into chunks of `chunk` tokens: parallel within a chunk, the
 * state carried serially between chunks ("Moonshot AI's New Attention
 * Architecture: Key Innovations Explained", sec. 3 Hardware-Friendly
 * Algorithm, the state recurrence and the output with its causal Tril).  Per
 * chunk the intra-chunk lower-triangular system A (the chunk Gram matrix of
 * the keys, gated and scaled by beta) is inverted by forward substitution,
 * T = (I + A)^-1, giving the WY factors W = T diag(beta) K_bar and
 * U = T diag(beta) V ("OSDN ...", sec. 2.1: the WY pipeline).  Gates are
 * cumulated in the log domain within each chunk (Moonshot page, sec. 5).
 *
 *   q, k          [B, T, H, Dk]  element type `dtype`
 *   v             [B, T, H, Dv]  element type `dtype`
 *   beta          [B, T, H]      element type `dtype`, the write strength
 *   g             log a_t <= 0: [B, T, H] (GDN_GATE_SCALAR) or [B, T, H, Dk]
 *                 (GDN_GATE_PER_DIM), element type `dtype`; must be NULL iff
 *                 gate_kind == GDN_GATE_NONE
 *   initial_state [B, H, Dk, Dv] fp32 (M = S^T), or NULL for a zero state
 *   o             [B, T, H, Dv]  element type `dtype` (output)
 *   final_state   [B, H, Dk, Dv] fp32 (output) or NULL; may be the same
 *                 pointer as initial_state (updated in place), any other
 *                 overlap with an input is GDN_ERR_INVALID_ARG
 *   B, T, H       batch, tokens per sequence, heads; T = 0 is allowed (no
 *                 output tokens; final_state = initial_state or 0); B = 0 or
 *                 H = 0 is a no-op
 *   Dk, Dv        64 or 128 each
 *   chunk         64
 *   dtype         GDN_BF16 (tensor-core path, fp32 accumulation and fp32
 *                 state) or GDN_F32 (fp32 CUDA-core path)
 *   workspace     device scratch of at least gdn_chunk_fwd_workspace_min_bytes
 *                 bytes, gdn_chunk_fwd_workspace_bytes for full speed (may be
 *                 NULL when the minimum is 0); workspace_bytes is its size
 * Returns GDN_OK once the work is enqueued.
 */
GDN_API gdn_status gdn_chunk_fwd(const void* q, const void* k, const void* v,
                         const void* beta, const void* g, gdn_gate gate_kind,
                         const float* initial_state, void* o, float* final_state,
                         int B, int T, int H, int Dk, int Dv, int chunk,
                         gdn_dtype dtype, void* workspace, size_t workspace_bytes,
                         gdn_stream_t stream);

/* Bytes of device workspace with which gdn_chunk_fwd runs fastest for these
 * arguments (0 when it needs none).  Returns (size_t)-1 for an unsupported or
 * invalid shape. */
GDN_API size_t gdn_chunk_fwd_workspace_bytes(int B, int T, int H, int Dk, int Dv, int chunk,
                                     gdn_dtype dtype, gdn_gate gate_kind);

/* Least workspace gdn_chunk_fwd accepts for these arguments (0 when it needs
 * none; never more than gdn_chunk_fwd_workspace_bytes).  Any size in between
 * works: the forward runs the sequence in waves of chunks whose step images
 * fit the workspace, so less workspace means shorter waves and less overlap,
 * with results identical to the bit -- except that with few (batch, head)
 * pairs and long waves the full-speed size also holds the buffers of the
 * segment-parallel state pass, which rounds differently (within the
 * tolerance); gdn_chunk_fwd_plan tells which.  Returns (size_t)-1 for an
 * unsupported or invalid shape. */
GDN_API size_t gdn_chunk_fwd_workspace_min_bytes(int B, int T, int H, int Dk, int Dv, int chunk,
                                                 gdn_dtype dtype, gdn_gate gate_kind);

/*
 * gdn_chunk_fwd_plan -- how gdn_chunk_fwd runs these arguments with
 * `workspace_bytes` of workspace (no device access, nothing enqueued):
 *   *waves            number of waves (launch groups) the sequence runs in
 *   *chunks_per_wave  chunks of every (batch, head) in a full wave
 *   *segments         segments per (batch, head) of a full wave: 1 is the
 *                     serial state pass; S > 1 is the segment-parallel pass
 *                     (each chunk maps the entering state affinely, so a run of
 *                     chunks does too: the offsets and transitions of all S
 *                     segments are formed in parallel, composed in order, and
 *                     every segment then runs from its own entering state;
 *                     "Moonshot AI's New Attention Architecture", sec. 3, the
 *                     chunkwise state recurrence).  Chosen when the (batch,
 *                     head) pairs leave most SMs idle and the workspace holds
 *                     its buffers (gdn_chunk_fwd_workspace_bytes does).
 * Returns GDN_ERR_WORKSPACE below gdn_chunk_fwd_workspace_min_bytes and the
 * argument errors of gdn_chunk_fwd_workspace_bytes.
 */
GDN_API gdn_status gdn_chunk_fwd_plan(int B, int T, int H, int Dk, int Dv, int chunk,
                                      gdn_dtype dtype, gdn_gate gate_kind,
                                      size_t workspace_bytes, int* waves, int* chunks_per_wave,
                                      int* segments);

/*
 * gdn_decode_step -- one recurrent step for N independent sequences: the
 * linear layers' constant-size-state decoding ("Moonshot AI's New Attention
 * Architecture", sec. 1) applied to the gated delta rule above.  Per (n, h):
 *     M' = Diag(a) M;  x = M'^T k;  r = beta (v - x);
 *     M  <- M' + k r^T (in place);  o = M^T q = M'^T q + r (k . q).
 * One pass over the state: each element is read once and written once.
 *
 *   q, k   [N, H, Dk]  element type `dtype`
 *   v      [N, H, Dv]  element type `dtype`
 *   beta   [N, H]      element type `dtype`
 *   g      [N, H] (scalar) or [N, H, Dk] (per-dimension), or NULL iff
 *          gate_kind == GDN_GATE_NONE
 *   state  [N, H, Dk, Dv] fp32, read and updated in place
 *   o      [N, H, Dv]  element type `dtype` (output; must not overlap state)
 *   N, H   >= 0 (0 is a no-op);  Dk, Dv in {64, 128}
 */
GDN_API gdn_status gdn_decode_step(const void* q, const void* k, const void* v,
                           const void* beta, const void* g, gdn_gate gate_kind,
                           float* state, void* o, int N, int H, int Dk, int Dv,
                           gdn_dtype dtype, gdn_stream_t stream);

/*
 * gdn_osdn_precondition -- phase 1 of the preconditioned delta rule: the
 * write keys kw_t = d_t (.) k_t of a diagonal preconditioner learned online
 * ("OSDN: Improving Delta Rule with Provable Online Preconditioning in Linear
 * Attention", sec. 2.1 the preconditioned key, sec. 2.2 the closed-form
 * surrogate and its online gradient step, sec. 2.3 the retention gate).  Per
 * (batch, head), token by token, with s = <d, k_t^2> and n = |k_t|^2:
 *     kw_t = d (.) k_t
 *     d   <- r_t d + eta beta_t (1 - beta_t s) k_t^2 / n     (unchanged if n = 0)
 * i.e. one step of gradient descent on h_t(d) = ((1 - beta_t <d, k_t^2>)^2 - 1)
 * / (2 |k_t|^2) after scaling d by r_t.  Phase 2 is gdn_chunk_fwd_wk with
 * these write keys.
 *
 *   k        [B, T, H, Dk]  element type `dtype`
 *   beta     [B, T, H]      element type `dtype`
 *   r        [B, T, H]      retention gate, element type `dtype`; NULL: r = 1
 *   eta      step size of the preconditioner (finite)
 *   d0       [B, H, Dk] fp32 initial preconditioner; NULL: all ones
 *   k_write  [B, T, H, Dk]  element type `dtype` (output; must not overlap
 *            any input)
 *   d_final  [B, H, Dk] fp32 final preconditioner (output) or NULL; may be
 *            the same pointer as d0
 *   Dk       64 or 128;  dtype GDN_BF16 or GDN_F32 (fp32 arithmetic either way)
 *   workspace, workspace_bytes: caller-owned device scratch of at least
 *            gdn_osdn_precondition_workspace_bytes(B, T, H, Dk) bytes (16-byte
 *            aligned, clear of every other argument); NULL / 0 when that is 0;
 *            less returns GDN_ERR_WORKSPACE before any launch.
 * The scan runs in blocks of 64 tokens: the step e_t = eta beta_t (1 - beta_t
 * s_t) / n_t is affine in s_t = <d_t, k_t^2>, so a block entering with d
 * solves a unit lower-triangular system through the Gram matrix of the k_t^2
 * (formed for every block at once); only a short pass per (batch, head) runs
 * the blocks in order (three launches).  Results equal the token-by-token scan
 * up to fp32 rounding.
 */
GDN_API gdn_status gdn_osdn_precondition(const void* k, const void* beta, const void* r,
                                         float eta, const float* d0, void* k_write,
                                         float* d_final, int B, int T, int H, int Dk,
                                         gdn_dtype dtype, void* workspace,
                                         size_t workspace_bytes, gdn_stream_t stream);
/* Workspace of gdn_osdn_precondition (bytes; (size_t)-1 for invalid sizes). */
GDN_API size_t gdn_osdn_precondition_workspace_bytes(int B, int T, int H, int Dk);

/*
 * gdn_chunk_fwd_wk -- gdn_chunk_fwd with a separate write key (phase 2 of the
 * preconditioned delta rule, "OSDN ...", sec. 2.1): per token
 *     M_t = (I - beta_t kw_t k_t^T) Diag(a_t) M_{t-1} + beta_t kw_t v_t^T,
 *     o_t = M_t^T q_t,
 * the residual read with k_t and written along kw_t.  Chunkwise, kw replaces
 * k in the Gram matrix and the intra-chunk scores (and in the state update);
 * k stays in the WY factor W.  Arguments as gdn_chunk_fwd plus
 *   k_write  [B, T, H, Dk] element type `dtype`, or NULL (then exactly
 *            gdn_chunk_fwd); with a write key the call runs on the
 *            tensor-core path only (GDN_BF16, Dk = Dv = 128), anything else is
 *            GDN_ERR_UNSUPPORTED.
 * Workspace as gdn_chunk_fwd (gdn_chunk_fwd_workspace_bytes / _min_bytes).
 */
GDN_API gdn_status gdn_chunk_fwd_wk(const void* q, const void* k, const void* k_write,
                                    const void* v, const void* beta, const void* g,
                                    gdn_gate gate_kind, const float* initial_state, void* o,
                                    float* final_state, int B, int T, int H, int Dk, int Dv,
                                    int chunk, gdn_dtype dtype, void* workspace,
                                    size_t workspace_bytes, gdn_stream_t stream);

/*
 * gdn_chunk_bwd -- gradients of gdn_chunk_fwd.  The pages print no backward;
 * the gradient is the derivative of the chunkwise forward ("Moonshot AI's New
 * Attention Architecture", sec. 3; the WY factors of "OSDN ...", sec. 2.1)
 * taken by hand.  The adjoint state dh = (gamma I + Phi^T) dh' + Qp^T dO runs
 * the transpose of the forward's affine chunk map from the last chunk back;
 * inside each chunk the products through T = (I + A)^-1, W, U, P and the
 * decays give the input gradients.  The call runs the forward again (one wave,
 * keeping its step images and every chunk's entering state), the adjoint
 * chain, then every chunk's gradients.
 *
 *   q, k, v, beta, g, gate_kind, initial_state   the forward's inputs (as
 *                 gdn_chunk_fwd; GDN_BF16, Dk = Dv = 128, gate none or scalar)
 *   d_o           [B, T, H, Dv] bf16, dL/do
 *   d_final_state [B, H, Dk, Dv] fp32, dL/dS_final, or NULL (zero)
 *   dq, dk        [B, T, H, Dk] fp32 (outputs)
 *   dv            [B, T, H, Dv] fp32 (output)
 *   dbeta         [B, T, H] fp32 (output)
 *   dg            [B, T, H] fp32 (output; NULL iff gate_kind == GDN_GATE_NONE)
 *   d_initial_state [B, H, Dk, Dv] fp32 (output) or NULL
 *   workspace     at least gdn_chunk_bwd_workspace_bytes bytes
 * Outputs must not overlap the inputs or one another.  Anything else than
 * bf16, d = 128 and a scalar gate or none is GDN_ERR_UNSUPPORTED.
 */
GDN_API gdn_status gdn_chunk_bwd(const void* q, const void* k, const void* v, const void* beta,
                                 const void* g, gdn_gate gate_kind, const float* initial_state,
                                 const void* d_o, const float* d_final_state, float* dq,
                                 float* dk, float* dv, float* dbeta, float* dg,
                                 float* d_initial_state, int B, int T, int H, int Dk, int Dv,
                                 int chunk, gdn_dtype dtype, void* workspace,
                                 size_t workspace_bytes, gdn_stream_t stream);

/* Workspace of gdn_chunk_bwd (the forward's images, its output, the entering
 * state and the adjoint of every chunk); (size_t)-1 for an unsupported shape. */
GDN_API size_t gdn_chunk_bwd_workspace_bytes(int B, int T, int H, int Dk, int Dv, int chunk,
                                             gdn_dtype dtype, gdn_gate gate_kind);

/* Synchronizes `stream`, then reads and clears the library's device status
 * word.  Returns GDN_ERR_TIMEOUT if any kernel since the last call gave up a
 * bounded wait, GDN_ERR_CUDA if the stream reports an error, else GDN_OK.
 * The status word's device address is looked up once per device ordinal and
 * cached; the cache does not survive cudaDeviceReset. */
GDN_API gdn_status gdn_read_device_status(gdn_stream_t stream);

/* A static, human-readable name for a status code. */
GDN_API const char* gdn_status_string(gdn_status s);

/*
 * gdn_chunk_fwd_noalloc -- gdn_chunk_fwd for callers that cannot allocate
 * device memory (no counterpart on the source pages: it is a deployment aid).
 *
 * Same arguments and results as gdn_chunk_fwd, minus the workspace: the
 * library supplies it from a fixed scratch array of
 * gdn_chunk_fwd_noalloc_scratch_bytes() bytes (128 MiB) that every GPU loading
 * the library reserves until the process exits.  For callers that cannot call
 * cudaMalloc -- inside a host framework that owns all device memory, or on a
 * path where allocation is forbidden.
 *   - No allocation: the call never calls cudaMalloc, cudaFree or any
 *     allocating library routine.
 *   - Limit: shapes whose gdn_chunk_fwd_workspace_min_bytes exceeds the
 *     scratch return GDN_ERR_WORKSPACE (nothing is enqueued); argument errors
 *     are reported exactly as by gdn_chunk_fwd.  Shapes whose
 *     gdn_chunk_fwd_workspace_bytes exceeds the scratch run with the waves
 *     the scratch allows.
 *   - Set-up: the array is reserved on a device when the library's module
 *     holding it is loaded there -- under lazy module loading (the CUDA
 *     default) on first use, not when the library is loaded.  A call with
 *     B = 0 or H = 0 (and otherwise valid sizes) does nothing but that
 *     set-up for the current device: it loads the module and looks up the
 *     array's device address (cudaGetSymbolAddress) with that device current,
 *     and returns GDN_OK, or GDN_ERR_CUDA if the device cannot hold the array.
 *     Make this call once per device at start-up, before the caller's
 *     framework reserves the device memory and before any stream capture;
 *     without it the first call with work does the set-up.  The looked-up
 *     address is cached per device ordinal and does not survive
 *     cudaDeviceReset.
 *   - Sharing: all calls on a device share the array and it keeps the last
 *     call's contents (the forward needs no cleared scratch).  Calls whose
 *     work overlaps on the GPU -- different streams, or unordered host
 *     threads -- race on it; order them on one stream.
 */
GDN_API gdn_status gdn_chunk_fwd_noalloc(const void* q, const void* k, const void* v,
                                         const void* beta, const void* g, gdn_gate gate_kind,
                                         const float* initial_state, void* o,
                                         float* final_state, int B, int T, int H, int Dk,
                                         int Dv, int chunk, gdn_dtype dtype,
                                         gdn_stream_t stream);

/* Size in bytes of the scratch array gdn_chunk_fwd_noalloc uses. */
GDN_API size_t gdn_chunk_fwd_noalloc_scratch_bytes(void);

/* Number of kernels this library has launched in this process (all devices,
 * all entry points), counted on the host at each successful launch. */
GDN_API unsigned long long gdn_kernel_launch_count(void);

/* Names of the kernels gdn_chunk_fwd launches for these arguments (comma
 * separated when it launches more than one), or NULL if the combination is
 * unsupported.  Static string; never freed. */
GDN_API const char* gdn_chunk_fwd_kernel_name(int Dk, int Dv, gdn_gate gate_kind,
                                              gdn_dtype dtype);

/* Library ABI version, currently 1. */
GDN_API int gdn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H */
