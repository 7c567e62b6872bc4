/*
 * m2rnn.h — C ABI of the B200 (sm_100a) M²RNN recurrence library (libm2rnn.so).
 *
 * The operation (per batch element b and head h, independently):
 *   Z_t = tanh(H_{t-1} W + k_t v_tᵀ)
 *   H_t = f_t H_{t-1} + (1 - f_t) Z_t
 *   y_t = H_tᵀ q_t
 * The first two lines are the state-update equations of "M²RNN: Non-Linear
 * RNNs with Matrix-Valued States for Scalable Language Modeling"
 * (gist.science technical summary, §2.1 core architecture design; also the
 * wispaper.ai post "M2 RNN: Breaking the Expressivity Ceiling of Linear RNNs
 * with Matrix-Valued States", §1 The Core Recurrence).  H_t is K×V, W is V×V
 * per head (it right-multiplies H_{t-1}; §2.2 gives the GEMM shape (K, V, V)),
 * f_t ∈ [0,1] is one scalar per (b, head, t) that depends on the input only.
 * The readout y_t = H_tᵀ q_t (q_t ∈ R^K, applied to the updated state) is
 * this library's reading: the pages define no readout.
 *
 * Layout: every tensor is dense, contiguous, head-first, row-major:
 *   k, q, dk, dq   [B][G][T][K]      v, y, dy   [B][H][T][V]      f, df  [B][H][T]
 *   W, dW  [H][V][V]         H0, HT, dHT, dH0  [B][H][K][V]
 *   ckpt   [B][H][ceil(T/C)][K][V]   (C = ckpt_stride; ckpt[.,.,c] = H_{c·C})
 * G = H unless k and q are grouped (m2rnn_dims.qk_heads): G groups of H/G
 * consecutive heads, head h reading the k and q of group h / (H/G), while
 * v, f, W and the state stay per head.  This is the library's reading of the
 * grouped-value form of the pages' tensor-parallel scheme (gist.science
 * §2.2: the topology-aware strategy needs no communication; the other one
 * all-reduces the gradients of the query and key that heads share).  dk and
 * dq of a group are the sums over its heads, in ascending head order.
 * Element types: in M2RNN_MODE_BF16_TC the inputs k, v, q, W, dy are bf16
 * (raw 16-bit words) and everything else is fp32.  In M2RNN_MODE_FP32_DEBUG
 * all tensors are fp32.
 *
 * Ownership and synchronisation: the caller allocates every buffer (device
 * memory) and the workspace; the library allocates nothing, keeps no state
 * between calls and never synchronises, except in m2rnn_get_device_status.
 * Calls are stream-ordered and asynchronous.  Outputs are overwritten, never
 * accumulated (dW is the sum over batch and time, written once).  All
 * pointers must be 16-byte aligned device pointers.
 *
 * Errors: argument problems return a status immediately and launch nothing.
 * Launch failures return M2RNN_ERR_CUDA.  Every wait inside a kernel is
 * bounded; a wait that runs out sets a status word in the workspace and the
 * kernel returns early (its outputs are then undefined); read it with
 * m2rnn_get_device_status.
 */
#ifndef M2RNN_H_
#define M2RNN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    M2RNN_OK = 0,
    M2RNN_ERR_INVALID_ARG = 1,       /* NULL required pointer, negative size, bad mode, qk_heads or f_is_logit */
    M2RNN_ERR_UNSUPPORTED_SHAPE = 2, /* K or V outside {16,32,64,128}, ckpt_stride < 1 */
    M2RNN_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned */
    M2RNN_ERR_WORKSPACE = 4,         /* workspace NULL or smaller than m2rnn_workspace_size */
    M2RNN_ERR_CUDA = 5,              /* a CUDA runtime call or kernel launch failed */
    M2RNN_ERR_DEVICE_TIMEOUT = 6     /* a bounded device-side wait ran out */
} m2rnn_status;

typedef enum {
    /* bf16 k/v/q/W inputs; the per-step H_{t-1}·W runs on the tcgen05 tensor
     * cores (bf16 operands, fp32 accumulation in tensor memory).  The fp32
     * state is fed to the MMA as a compensated pair of bf16 operands
     * (hi + lo), so the operand carries about 16 bits of mantissa; a
     * forward that writes checkpoints (ckpt != NULL) feeds it as three bf16
     * terms (about 24 bits) and evaluates tanh with a small relative error
     * near zero as well, since the backward's gradients can amplify the
     * checkpoints' relative error (heads whose W has a spectral radius above
     * 1).  y and H_T of the two kinds of call therefore agree to rounding,
     * not bit for bit. */
    M2RNN_MODE_BF16_TC = 0,
    /* fp32 everything, CUDA-core FFMA and accurate tanhf: a slow reference
     * mode on the device. */
    M2RNN_MODE_FP32_DEBUG = 1,
    /* As M2RNN_MODE_BF16_TC, but tanh is the single-SFU tanh.approx.f32
     * (about 2^-11 relative error per element instead of about 1e-6
     * absolute): a faster forward for inference, where y and H_T stay well
     * inside the tensor-core mode's tolerance.  Forward only: m2rnn_backward
     * returns M2RNN_ERR_INVALID_ARG and m2rnn_workspace_size(d, 1) returns 0
     * (gradients over long sequences amplify the tanh error). */
    M2RNN_MODE_BF16_TC_FAST_TANH = 2,
    /* bf16 inputs, forward only, V = 64 and K in {16, 32, 64} (other shapes
     * return M2RNN_ERR_UNSUPPORTED_SHAPE): a latency-oriented alternative
     * forward with the state resident in registers (warp-level mma.sync, 16
     * rows per warp, no per-step barrier).  Same compensated pair as
     * M2RNN_MODE_BF16_TC, with the tanh that is accurate near zero in
     * relative terms; its checkpoints may be passed to
     * m2rnn_backward in M2RNN_MODE_BF16_TC.  m2rnn_backward rejects this mode
     * (M2RNN_ERR_INVALID_ARG). */
    M2RNN_MODE_BF16_MMA_SYNC = 3
} m2rnn_mode;

typedef struct {
    int B, H, T, K, V;  /* batch, heads, steps, state rows (key dim), state columns (value dim) */
    int mode;           /* m2rnn_mode */
    int ckpt_stride;    /* C >= 1: the forward stores H_{c·C} for the backward */
    int qk_heads;       /* G, the head groups of k and q: 0 (or H) = one per head;
                         * otherwise 1 <= G < H with H % G == 0, else
                         * M2RNN_ERR_INVALID_ARG */
    int f_is_logit;     /* 0: f holds the gate f_t in [0, 1].  1: f holds gate
                         * logits a_t and f_t = 1 / (1 + exp(-a_t)), evaluated
                         * in the kernels (accurate expf); m2rnn_backward then
                         * writes dL/da_t = dL/df_t · f_t (1 - f_t) to df.
                         * Other values: M2RNN_ERR_INVALID_ARG.  The library's
                         * reading of the gate parameterisation ψ(x_t) (gist.science
                         * §2.1 forget gate): ψ ends in the logistic function;
                         * how a_t comes from x_t (a projection, a per-head bias
                         * setting each head's initial decay) is the caller's. */
} m2rnn_dims;

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* m2rnn_stream_t;

/* Bytes of device workspace a call needs (forward when backward == 0).
 * Returns 0 for invalid dims.  The first 256 bytes hold the device status
 * word: zero them once after allocating the workspace.  The rest is scratch
 * the kernels write before they read it: for the backward, per-(b, h) dW
 * partials and, except for V = 64 with a stride of at most 8 (16 for
 * K = 32), whose chunk stays on chip, the chunk recompute buffer, plus,
 * when k and q are grouped,
 * the per-head dk and dq (2 · B·H·T·K fp32) summed into the groups' dk and
 * dq at the end, and, when V = 128 with K >= 64 (rows split over several
 * CTAs per pair), the slices' dv and df partials (slices · B·H·T·(V+1) fp32);
 * for a bf16 forward with few (b, h) pairs, which splits each pair's K rows
 * over several CTAs (K/8 slices when V = 64 and B·H·K/8 <= 148, else up to 8
 * slices when B·H·2 <= 148), the slices' partial readouts (slices · B·H·T·V
 * fp32). */
size_t m2rnn_workspace_size(const m2rnn_dims* d, int backward);

/* Forward scan.  H0 may be NULL (zero initial state).  HT (final state) and
 * ckpt (checkpoints for m2rnn_backward) may be NULL.  y is required.
 * H0 and HT may be the same buffer: every element of H0 is read before the
 * same element of HT is written, so the state can be advanced in place --
 * with T = 1 this is one decode step, and T such calls give the scan's y and
 * H_T bit for bit.  This is the library's single-step decode: there is no
 * separate step entry point (the Python binding's step() is this call with
 * T = 1 and H0 == HT). */
m2rnn_status m2rnn_forward(const m2rnn_dims* d,
                           const void* k, const void* v, const void* q,
                           const float* f, const void* W, const float* H0,
                           float* y, float* HT, float* ckpt,
                           void* workspace, size_t ws_bytes, m2rnn_stream_t stream);

/* Backward through time for the loss L with dL/dy = dy and dL/dH_T = dHT
 * (NULL = 0; dHT and dH0 may be the same buffer).  ckpt must come from
 * m2rnn_forward with the same inputs and
 * the same dims (including ckpt_stride); the states inside each chunk of C
 * steps are recomputed from it.  The initial state H_0 is not an argument:
 * it is ckpt[b][h][0], which m2rnn_forward writes from its H0 (zeros for a
 * NULL H0), so the recomputation always starts from the state the forward
 * used and a second copy of H_0 cannot disagree with the checkpoints.  Writes dk, dv, dq, df, dW, dH0 (all
 * required, all fp32).  M2RNN_MODE_BF16_TC supports every K, V in
 * {16, 32, 64, 128} with ckpt_stride <= 16 (a longer stride returns
 * M2RNN_ERR_UNSUPPORTED_SHAPE); for V = 64 and K >= 32 a stride of at most 8
 * (16 for K = 32) takes the faster kernel, which keeps the recomputed chunk
 * on chip.  M2RNN_MODE_FP32_DEBUG supports every stride. */
m2rnn_status m2rnn_backward(const m2rnn_dims* d,
                            const void* k, const void* v, const void* q,
                            const float* f, const void* W, const float* ckpt,
                            const void* dy, const float* dHT,
                            float* dk, float* dv, float* dq, float* df,
                            float* dW, float* dH0,
                            void* workspace, size_t ws_bytes, m2rnn_stream_t stream);

/* Allocation-free m2rnn_backward (the pages describe no such variant: it is
 * an interface addition of this library).  For callers that cannot allocate
 * device memory when they need gradients: services that forbid allocator
 * calls after start-up (an allocation can synchronise the device or fail
 * under memory pressure) and hosts that hand the library only the tensors
 * they already own.  Same arguments and results (bit for bit) as
 * m2rnn_backward minus the workspace: the scratch comes from a 32 MiB array
 * compiled into the library, which every GPU that loads the library keeps
 * until the process exits.
 *  - Problems with m2rnn_workspace_size(d, 1) > 32 MiB return
 *    M2RNN_ERR_WORKSPACE and launch nothing.
 *  - All calls share the array: calls whose kernels overlap on the GPU race
 *    and give wrong results; order them on one stream.
 *  - The first call on a device looks up the array's device address (no
 *    allocation); make it before any stream capture starts.  The address is
 *    cached per device for the life of the process: do not use this entry
 *    point across a device reset.
 *  - Device-side wait timeouts are not reported by this entry point. */
m2rnn_status m2rnn_backward_noalloc(const m2rnn_dims* d,
                                    const void* k, const void* v, const void* q,
                                    const float* f, const void* W, const float* ckpt,
                                    const void* dy, const float* dHT,
                                    float* dk, float* dv, float* dq, float* df,
                                    float* dW, float* dH0, m2rnn_stream_t stream);

/* Synchronises `stream`, reads and clears the status word in `workspace`.
 * Returns M2RNN_OK or M2RNN_ERR_DEVICE_TIMEOUT (or M2RNN_ERR_CUDA). */
m2rnn_status m2rnn_get_device_status(void* workspace, m2rnn_stream_t stream);

/* Static, human-readable name of a status code. */
const char* m2rnn_status_string(m2rnn_status s);

/* Upper bound, in nanoseconds, for every device-side wait of later launches
 * (default 2e9).  Values below 1e5 are raised to 1e5. */
void m2rnn_set_wait_limit_ns(uint64_t ns);

/* Test hook: host-side fault injection for later launches (not part of the
 * method).  0 = none; 1 = the input producer of the bf16 forward (tensor-core
 * or row kernel) and of the tensor-core backwards stops after its first chunk
 * (16 steps forward, one checkpoint chunk backward), so the kernel's bounded
 * waits run out: the
 * call returns M2RNN_OK, the kernel exits early with undefined outputs and
 * m2rnn_get_device_status reports M2RNN_ERR_DEVICE_TIMEOUT (after about the
 * wait limit).  Returns M2RNN_OK, or M2RNN_ERR_INVALID_ARG for other values. */
int m2rnn_debug_set_fault(int fault);

#ifdef __cplusplus
}
#endif

#endif /* M2RNN_H_ */
