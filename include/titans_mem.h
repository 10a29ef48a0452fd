/*
 * titans_mem.h -- C ABI of the Titans neural long-term memory library (sm_100a).
 *
 * The library computes the chunk-wise forward pass of the neural long-term
 * memory described in "Titans: Learning to Memorize at Test Time" (pages: the
 * mer.dev walk-through, sec. 3.1-3.2; the lowest.today German summary,
 * "Gedaechtnisaktualisierungsmechanismus"; the hotdry blog, sec. 3.1):
 *
 *   memory      linear  M(x) = W x                 (walk-through sec. 3.1 "Memory Architecture")
 *               MLP     M(x) = W2 silu(W1 x)       (blog sec. 3.1; SiLU per sec. 4.4)
 *   loss        l_t = || M(k_t) - v_t ||_2^2       (sec. 3.1 "Objective")
 *   momentum    S_t = eta_t S_{t-1} - theta_t grad l_t      (sec. 3.1 "Surprise Metric")
 *   forgetting  M_t = (1 - alpha_t) M_{t-1} + S_t           (sec. 3.1 "Forgetting Mechanism")
 *   chunking    every token of a chunk of b tokens takes its gradient at the
 *               weights the chunk started with (sec. 3.2, t' = t - mod(t, b))
 *   retrieval   y_t = M*(q_t), a forward pass with no update, using the same
 *               chunk-start weights (sec. 3.1 "Retrieving a Memory")
 *
 * One "unit" is one (batch, head) pair; units are independent.
 *
 * Conventions for every call:
 *  - Tensors are DEVICE pointers, row-major, contiguous, owned by the caller;
 *    the library never frees or retains them. k, q, v, y and the state are
 *    16-byte aligned; the gates alpha, eta, theta 4-byte aligned.
 *  - Calls are asynchronous on the caller's CUDA stream (passed as void*, a
 *    cudaStream_t; NULL = the legacy default stream).
 *  - Argument checks happen before any launch and return TITANS_EINVAL or
 *    TITANS_EUNSUPPORTED with a message in titans_last_error_string(); a
 *    launch failure returns TITANS_ECUDA. Faults a kernel detects itself
 *    (a wait that ran out of time) are recorded in a device status word that
 *    titans_mem_sync_status() reads and clears (TITANS_EDEVICE).
 *  - The calls allocate no device memory; titans_mem_init allocates the
 *    handle's workspace and status word once.
 *  - k and q are expected l2-normalised by the caller (sec. 4.4); the library
 *    does not normalise.
 */
#ifndef TITANS_MEM_H
#define TITANS_MEM_H

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TITANS_OK = 0,
    TITANS_EINVAL = 1,        /* bad argument: null/misaligned pointer, bad size */
    TITANS_EUNSUPPORTED = 2,  /* valid but not supported (dimension, chunk length) */
    TITANS_ECUDA = 3,         /* a CUDA runtime call or launch failed */
    TITANS_EDEVICE = 4        /* the device status word reported a fault (timeout) */
} titans_status_t;

typedef enum {
    TITANS_BF16 = 0,  /* k, q, v, y bf16; tensor-core arithmetic with fp32 accumulate; fp32 state */
    TITANS_FP32 = 1   /* k, q, v, y fp32; CUDA-core fp32 arithmetic; fp32 state (reference mode) */
} titans_mode_t;

/* flags */
#define TITANS_FLAG_CUDA_CORES 1u  /* run the CUDA-core chunk kernel even where the tensor-core one applies */
/* Chunk-shared gates (walk-through sec. 3.2, "Parameters as the Function of Chunks": alpha, eta,
 * theta shared by the tokens of a chunk make the memory's recurrence time-invariant inside the
 * chunk): the chunked forward calls then take alpha, eta, theta as [B, H, ceil(T / chunk)], one
 * value per chunk of the call, applied to each of the chunk's tokens (a ragged last chunk too).
 * titans_mem_step and titans_mem_forward_noalloc keep per-token gates. */
#define TITANS_FLAG_CHUNK_GATES 2u
/* Linear memory only: run the chunks by a cross-chunk scan instead of one after another. One
 * chunk of the linear memory is an affine map of [W | S], so segments of chunks compose their
 * maps in parallel, a short scan over the segments gives each segment's start state, and the
 * segments then run their chunks in parallel (the associative scan of the German summary's
 * "Parallelisiertes Training" and the tencent review). A handle spreads a unit over about
 * (SMs / units) segments, which pays for long streams of few units. fp32 arithmetic. */
#define TITANS_FLAG_CHUNK_SCAN 4u

typedef struct {
    int d;             /* key/value width: 64 or 128 */
    int d_hidden;      /* MLP hidden width h (4*d); 0 = linear memory */
    int chunk;         /* largest chunk length the handle will be asked for, 1..128 */
    titans_mode_t mode;
    int B, H;          /* batch and heads: B*H units */
    unsigned flags;    /* TITANS_FLAG_* */
} titans_mem_config;

typedef struct titans_mem *titans_mem_t;

/* Kernel a call would run (titans_mem_path). */
typedef enum {
    TITANS_PATH_TC_MLP64 = 1,     /* tcgen05 bf16 chunk kernel, d=64, h=256, chunk<=64 */
    TITANS_PATH_CUDA_CORES = 2,   /* CUDA-core fp32 chunk kernel (any supported shape) */
    TITANS_PATH_STEP_CLUSTER = 3, /* single-token decode, thread-block-cluster kernel (MLP) */
    TITANS_PATH_TC_PHASED = 4,    /* tcgen05 bf16 chunk kernel over all SMs, d=128, h=512, chunk<=128 */
    TITANS_PATH_DEEP_CUDA_CORES = 5, /* deep memory (titans_mem_init_deep), CUDA-core chunk kernel */
    TITANS_PATH_LINEAR_SCAN = 6,     /* linear memory, cross-chunk scan (TITANS_FLAG_CHUNK_SCAN) */
    TITANS_PATH_TC_DEEP = 7,         /* deep memory, tcgen05 bf16 phased kernel over all SMs (L >= 3) */
    TITANS_PATH_TC_BACKWARD = 8      /* backward, tcgen05 bf16, one CTA per unit (d=64, h=256, chunk<=64) */
} titans_path_t;

/* Validates the configuration and allocates the handle, its device status word and
 * (for the CUDA-core path) its workspace on the current device.
 * Returns TITANS_EINVAL for a null pointer or a non-positive size,
 * TITANS_EUNSUPPORTED for d not in {64, 128}, d_hidden not in {0, 4d} or chunk
 * outside 1..128, TITANS_ECUDA if an allocation fails. */
titans_status_t titans_mem_init(const titans_mem_config *cfg, titans_mem_t *out);

/* titans_mem_init for a deep memory of `layers` layers (2..8), every hidden layer d_hidden wide:
 *   M(x) = W_L silu(W_{L-1} ... silu(W_1 x)),  no bias.
 * Defined by the walk-through's sec. 3.1 "Memory Architecture" (an MLP memory with L_M >= 2
 * layers, deeper ones strictly more expressive than the linear one) and sec. 5.5 "The Effect of
 * Deep Memory" (more layers remember better and cost throughput). Such a handle runs
 * titans_mem_forward_deep only. Returns TITANS_EUNSUPPORTED for layers outside 2..8, TITANS_EINVAL
 * for d_hidden = 0, and otherwise what titans_mem_init returns. */
titans_status_t titans_mem_init_deep(const titans_mem_config *cfg, int layers, titans_mem_t *out);

/* Frees the handle and its device memory. Must not race with work in flight. */
titans_status_t titans_mem_destroy(titans_mem_t m);

/*
 * Chunk-wise forward over T tokens of every unit (update + retrieve).
 * Defined by the walk-through's sec. 3.2 "How to Parallelize the Long-term Memory Training"
 * (chunks of b tokens; every token's gradient at the chunk-start weights, t' = t - mod(t, b);
 * the tensorized mini-batch form, here extended with the momentum term) applied to the
 * update of sec. 3.1 ("Surprise Metric": S_t = eta_t S_{t-1} - theta_t grad l(M_{t-1}; x_t);
 * "Forgetting Mechanism": M_t = (1 - alpha_t) M_{t-1} + S_t; "Objective": l = ||M(k) - v||^2)
 * and the retrieval y_t = M*(q_t) of sec. 3.1 "Retrieving a Memory".
 *   k, q, v     [B, H, T, d]  bf16 (TITANS_BF16) or fp32 (TITANS_FP32)
 *   alpha, eta, theta [B, H, T] fp32; alpha in [0, 1], eta, theta >= 0
 *   MLP state:  W1, S1 [B, H, h, d], W2, S2 [B, H, d, h] fp32;
 *   linear:     W1 = W, S1 = S [B, H, d, d] fp32, W2 = S2 = NULL
 *               (column convention M(k) = W k, W is [d_out, d_in]).
 *   The state is read at entry and overwritten with the state after token T-1.
 *   y           [B, H, T, d] same dtype as k: y_t = M(q_t) with the weights at the
 *               start of t's chunk.
 *   chunk       1..cfg->chunk; a last chunk shorter than `chunk` follows the same rules.
 * T >= 1 and T * d < 2^31 per unit.
 */
titans_status_t titans_mem_forward(titans_mem_t m, const void *k, const void *q, const void *v,
                                   const float *alpha, const float *eta, const float *theta,
                                   long T, int chunk, float *W1, float *W2, float *S1, float *S2,
                                   void *y, void *stream);

/*
 * titans_mem_forward with the memory-as-a-gate output in place of y:
 *   o_t = attn_t * sigmoid(M(q_t)), element-wise,
 * where attn [B, H, T, d] (dtype of k, 16-byte aligned, read only) is the output of the
 * layer's attention branch, computed by the caller, and M(q_t) is the retrieval that
 * titans_mem_forward writes as y. The update of the state is unchanged.
 * Defined by the walk-through's sec. 4.2 "Gated Memory" (o = y (x) M(x~), y the sliding-window
 * attention output) with the tencent review's MAG bullet (the combination is an element-wise
 * product with a non-linear activation); the reading taken is the logistic function of the
 * memory's retrieval gating the attention output. The gate is fused into the kernels' output
 * stores: o costs no extra pass over memory beyond reading attn.
 * Returns what titans_mem_forward returns, and TITANS_EINVAL for a NULL or misaligned attn.
 */
titans_status_t titans_mem_forward_gated(titans_mem_t m, const void *k, const void *q, const void *v,
                                         const float *alpha, const float *eta, const float *theta,
                                         long T, int chunk, float *W1, float *W2, float *S1, float *S2,
                                         const void *attn, void *o, void *stream);

/*
 * Chunk-wise forward of a deep memory (handle from titans_mem_init_deep; the same update and
 * retrieval rules as titans_mem_forward, sec. 3.1-3.2, applied to every layer).
 *   W, S  [B, H, P] fp32, P = 2 h d + (L - 2) h^2: per unit the layers one after another, each
 *         row-major [out][in]: W_1 [h][d], W_2 .. W_{L-1} [h][h], W_L [d][h]; read at entry and
 *         overwritten with the state after token T-1.
 *   attn  NULL for y = M(q), or the attention branch's output for the memory-as-a-gate output
 *         y = attn * sigmoid(M(q)) (see titans_mem_forward_gated).
 *   Other arguments as in titans_mem_forward. In TITANS_BF16 mode with 3..8 layers, chunk <= 128 and
 *   no TITANS_FLAG_CUDA_CORES it runs the tensor-core phased kernel (bf16 operands, fp32
 *   accumulation and state; TITANS_PATH_TC_DEEP); otherwise the CUDA-core chunk kernel (fp32
 *   arithmetic; k, q, v, y in the handle's dtype).
 */
titans_status_t titans_mem_forward_deep(titans_mem_t m, const void *k, const void *q, const void *v,
                                        const float *alpha, const float *eta, const float *theta,
                                        long T, int chunk, float *W, float *S, const void *attn, void *y,
                                        void *stream);

/* Device buffers that titans_mem_forward_host stages through, each the size of the host
 * array of the same name ([B, H, T, d] for k, q, v, y; [B, H, T] for the gates). The call
 * overwrites them; their contents afterwards are unspecified (segment-major layout). */
typedef struct {
    void *k, *q, *v;
    float *alpha, *eta, *theta;
    void *y;
} titans_device_buffers;

/*
 * titans_mem_forward with the token streams and y in HOST memory and the state on the
 * device: the gates are copied whole first, then T is cut into segments of t_seg tokens (a multiple of `chunk`; 0 picks about
 * five segments), and each segment's host-to-device copy, forward and device-to-host copy
 * of y run on three streams, so the copies of one segment overlap the compute and copies of
 * the others. Running a stream in segments gives exactly the result of one call over T (a
 * segment boundary is a chunk boundary).
 *   k, q, v, alpha, eta, theta, y: host arrays with titans_mem_forward's shapes and dtypes;
 *     page-locked memory (cudaHostAlloc / cudaHostRegister) lets the copies overlap, pageable
 *     memory is correct but serialises them. They must stay valid until `stream` completes.
 *   W1, W2, S1, S2: device state as in titans_mem_forward.
 *   dev: device scratch (see titans_device_buffers), 16-byte aligned like the device
 *     arguments of titans_mem_forward.
 * Asynchronous on `stream`: the copies start after the work already queued on it, and work
 * queued on it afterwards starts after the last copy of y. The handle's two copy streams are
 * created on first use; calls on one handle must not overlap.
 * Returns TITANS_EINVAL for a null pointer, a misaligned device buffer or a t_seg that is
 * not a multiple of chunk, TITANS_ECUDA if a copy or launch fails, and otherwise what
 * titans_mem_forward returns per segment. After an error, copies and segments queued
 * before it may still run; the call has made `stream` wait for them, so synchronize
 * `stream` before freeing or reusing the buffers.
 */
titans_status_t titans_mem_forward_host(titans_mem_t m, const void *k, const void *q, const void *v,
                                        const float *alpha, const float *eta, const float *theta,
                                        long T, int chunk, float *W1, float *W2, float *S1, float *S2,
                                        void *y, const titans_device_buffers *dev, long t_seg,
                                        void *stream);

/*
 * One decode step per unit with chunk = 1 semantics: y = M(q; W_{t-1}), then the
 * update with the gradient at W_{t-1}. Defined by the walk-through's sec. 3.1: the
 * per-token recurrence ("Surprise Metric", "Forgetting Mechanism", "Objective") and the
 * retrieval of "Retrieving a Memory", read with the previous token's memory as the MAC
 * variant's M*_{t-1} (sec. 4.1); it is sec. 3.2's chunked form with b = 1.
 *   k, q, v [B, H, d] (dtype of the mode); alpha, eta, theta [B, H] fp32;
 *   state as in titans_mem_forward, updated in place; y [B, H, d].
 */
titans_status_t titans_mem_step(titans_mem_t m, const void *k, const void *q, const void *v,
                                const float *alpha, const float *eta, const float *theta,
                                float *W1, float *W2, float *S1, float *S2, void *y, void *stream);

/* titans_mem_step with the memory-as-a-gate output o = attn * sigmoid(M(q; W_{t-1})) in place of
 * y; attn [B, H, d] in the dtype of k, 16-byte aligned (see titans_mem_forward_gated). */
titans_status_t titans_mem_step_gated(titans_mem_t m, const void *k, const void *q, const void *v,
                                      const float *alpha, const float *eta, const float *theta,
                                      float *W1, float *W2, float *S1, float *S2, const void *attn,
                                      void *o, void *stream);

/*
 * Chunk-wise forward that allocates no device memory, for callers that cannot call
 * cudaMalloc: code inside someone else's stream capture, under an allocator that owns all
 * device memory, on a path that must not synchronize the device, or a plug-in that must
 * not leave allocations behind (titans_mem_init allocates, so those callers cannot hold a
 * handle). The pages on the method have no counterpart: this is a deployment variant.
 *
 * Same arguments and semantics as titans_mem_forward, with the configuration passed
 * directly. cfg->flags and cfg->chunk are ignored: `chunk` may be any length in 1..128.
 * It always runs the CUDA-core (fp32 arithmetic) chunk kernel, never the tensor-core one,
 * so its results equal, bit for bit, those of titans_mem_forward on that kernel (fp32
 * mode, or TITANS_FLAG_CUDA_CORES). Its scratch is a fixed 16 MiB device array inside the
 * library, held by every GPU that loads the library until the process exits:
 *  - the first call on a device looks up the array there and loads the kernel's code for
 *    both modes; make it before any stream capture meant to contain later calls;
 *  - every call shares the array, so calls that overlap on a GPU race: serialize them;
 *  - nothing in the array needs clearing between calls;
 *  - a call needing more than the array holds -- B*H units x (4*chunk*h + chunk*d floats
 *    for the MLP memory, chunk*d for the linear one, each rounded up to 64 floats) -- returns
 *    TITANS_EUNSUPPORTED with a message in titans_last_error_string(); B*H above 2^30
 *    returns TITANS_EINVAL.
 * No device status word: the kernel has no waits to time out.
 */
titans_status_t titans_mem_forward_noalloc(const titans_mem_config *cfg, const void *k, const void *q,
                                           const void *v, const float *alpha, const float *eta,
                                           const float *theta, long T, int chunk, float *W1, float *W2,
                                           float *S1, float *S2, void *y, void *stream);

/*
 * Backward of the chunk-wise forward (the outer loop of training: the walk-through's sec. 3.1
 * makes the projections that produce k, v, q outer-loop parameters; the memory's forward is
 * defined by sec. 3.1-3.2), for the linear and the 2-layer MLP memory. For
 *   L = <dy, y> + <dW1, W1_T> + <dW2, W2_T> + <dS1, S1_T> + <dS2, S2_T>,
 * with y and the final state those of titans_mem_forward on the same inputs and initial state
 * (W1, W2, S1, S2 as in titans_mem_forward, read only; W2, S2, dW2, dS2, dW2_0, dS2_0 NULL for
 * the linear memory), it writes
 *   dk, dq, dv  [B, H, T, d] (dtype of k)      dL/dk, dL/dq, dL/dv
 *   dalpha, deta, dtheta [B, H, T] fp32        dL/d the gates
 *   dW1_0, dW2_0, dS1_0, dS2_0 (shapes of W1..S2) fp32  dL/d the initial state
 * from the upstream dy [B, H, T, d] (dtype of k) and dW1, dW2, dS1, dS2 (NULL = zero). It reruns
 * the forward, keeping every chunk-start state in `workspace` (caller-owned device memory of at
 * least titans_mem_backward_workspace_bytes(m, T, chunk) bytes, 16-byte aligned), then walks the
 * chunks backwards; the MLP's adjoint includes the second-order terms of the inner gradient.
 * In TITANS_BF16 mode with d = 64, h = 256, chunk <= 64 and no TITANS_FLAG_CUDA_CORES it runs on
 * tensor cores (titans_mem_path(m, chunk, 2) == TITANS_PATH_TC_BACKWARD): the forward is the
 * tensor-core chunk kernel writing checkpoints (its y goes to dk, which is then overwritten), and
 * the backward pass is bf16 tcgen05 GEMMs with fp32 accumulation. Otherwise fp32 on CUDA cores.
 * Per-token gates only. Returns TITANS_EUNSUPPORTED for a deep memory or with
 * TITANS_FLAG_CHUNK_GATES, TITANS_EINVAL for a NULL or misaligned pointer or a small workspace.
 */
size_t titans_mem_backward_workspace_bytes(titans_mem_t m, long T, int chunk);
titans_status_t titans_mem_backward(titans_mem_t m, const void *k, const void *q, const void *v,
                                    const float *alpha, const float *eta, const float *theta, long T,
                                    int chunk, const float *W1, const float *W2, const float *S1,
                                    const float *S2, const void *dy, const float *dW1, const float *dW2,
                                    const float *dS1, const float *dS2, void *dk, void *dq, void *dv,
                                    float *dalpha, float *deta, float *dtheta, float *dW1_0,
                                    float *dW2_0, float *dS1_0, float *dS2_0, void *workspace,
                                    size_t workspace_bytes, void *stream);

/* Kernel that titans_mem_forward (step = 0), titans_mem_step (step = 1) or titans_mem_backward
 * (step = 2) would run with this chunk length; negative on an unsupported combination. */
int titans_mem_path(titans_mem_t m, int chunk, int step);

/* Synchronises the stream, then reads and clears the handle's device status word.
 * TITANS_OK if no kernel reported a fault since the last call, else TITANS_EDEVICE. */
titans_status_t titans_mem_sync_status(titans_mem_t m, void *stream);

/* Thread-local message for the last non-OK status returned on this thread. */
const char *titans_last_error_string(void);

/* Library version: major * 10000 + minor * 100 + patch. */
int titans_mem_version(void);

/* Diagnostic: the two evaluations of the MLP memory's activation that the tensor-core chunk kernel
 * uses, silu(z) = h (1 + tanh h) with h = z / 2 ("Titans", walk-through sec. 3.1: the memory is an
 * MLP; hotdry blog sec. 3.1: memory(x) = W2 sigma(W1 x) with SiLU). For each of the n fp32 values h
 * (device memory), silu_fma[i] takes tanh from fp32 arithmetic on the FMA pipe (Chebyshev
 * interpolants, absolute error on tanh below 1.1e-4) and silu_mufu[i] from the hardware's
 * tanh.approx. All three arrays are caller-owned device memory of n floats, asynchronous on
 * `stream`. TITANS_EINVAL for n < 0 or a NULL pointer, TITANS_ECUDA for a failed launch. */
titans_status_t titans_silu_routes(const float *h, float *silu_fma, float *silu_mufu, long n, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* TITANS_MEM_H */
