/*
 * m3.h -- C ABI of the Mamba-3 selective-SSM core on NVIDIA B200 (sm_100a).
 *
 * The operation is the recurrence of "Mamba-3: Improved Sequence Modeling using State Space
 * Principles": the exponential-trapezoidal update (Sec. 3.1.1, Prop. 1)
 *     h_t = alpha_t h_{t-1} + beta_t B_{t-1} x_{t-1}^T + gamma_t B_t x_t^T,
 *     alpha_t = exp(dt_t A_t), beta_t = (1 - lam_t) dt_t alpha_t, gamma_t = lam_t dt_t,
 * over a complex diagonal state realised as a cumulative data-dependent rotation of B and C
 * (Sec. 3.2.1 Prop. 2, Sec. 3.2.2 Prop. 4 and Appendix B.3: Bbar_t = (prod_{s<=t} R_s^T) B_t,
 * R_s = Block{R(dt_s theta_s[i])}), with B and C RMS-normalised and biased per head
 * (Sec. 3.4), in single-input (rank R = 1) and rank-R MIMO form (Sec. 3.3, Appendix C:
 * H_t = a_t H_{t-1} + B_t X_t^T, Y_t = H_t^T C_t), with y_t = H_t^T Cbar_t.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers to contiguous row-major buffers owned by the
 *    caller, 16-byte aligned. The library never allocates or frees device memory, never
 *    synchronises the device, and launches only on the given stream (a cudaStream_t passed
 *    as void*; NULL = the legacy default stream).
 *  - The complex state of size N/2 is stored as [Re; Im] halves: rotation pair i is
 *    (i, i + N/2) (Prop. 2: B = [B; B_hat]).
 *  - Head h reads B/C group h / (H / G).
 *  - Errors: an invalid argument returns M3_ERR_INVALID_ARG, a valid but unsupported shape
 *    M3_ERR_UNSUPPORTED, both before anything is launched; a launch failure returns
 *    M3_ERR_CUDA. m3_last_error() describes the most recent failure of the calling thread.
 *    No C++ exception crosses this interface.
 *  - Inputs that hold NaN or Inf propagate into the affected (batch, head) outputs only.
 */
#ifndef M3_H_
#define M3_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define M3_API __attribute__((visibility("default")))
#else
#define M3_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    M3_OK = 0,
    M3_ERR_INVALID_ARG = 1,
    M3_ERR_UNSUPPORTED = 2,
    M3_ERR_CUDA = 3,
    M3_ERR_TIMEOUT = 4
} m3_status;

/* Storage type of x, B, C, theta, y, prev_B and prev_x. dt, A, lam, the biases and the
 * state's h and phi are always fp32. */
typedef enum { M3_F32 = 0, M3_BF16 = 1 } m3_dtype;

typedef struct {
    int64_t batch;    /* b >= 0                                                     */
    int64_t seqlen;   /* L >= 0 (m3_decode_step: must be 1)                         */
    int64_t nheads;   /* H >= 1                                                     */
    int64_t ngroups;  /* G >= 1, H % G == 0: heads that share one B/C              */
    int64_t headdim;  /* P in {16, 32, 64, 128}                                    */
    int64_t dstate;   /* N, a multiple of 16, <= 256                               */
    int64_t rank;     /* R in {1, 2, 4, 8}; 1 = SISO                                */
    int64_t chunk;    /* tokens per chunk of the prefill scan (chunk * R <= 128;
                         64 or 128 rows run on the tensor cores, see m3_scan_fwd)  */
    int32_t in_dtype; /* m3_dtype                                                   */
    int32_t bc_norm;  /* nonzero: RMS-normalise B and C over N before the bias      */
    float norm_eps;   /* epsilon of the RMS norm (1e-6 is the usual value)          */
    uint32_t flags;   /* M3_DT_SOFTPLUS | M3_LAM_SIGMOID | M3_DISC_ZOH, or 0        */
} m3_dims;

/* m3_dims.flags: the step scalars arrive as the layer's raw projections and the kernels
 * apply the parameterisation themselves (the fused scalar prologue), per token and head:
 *   M3_DT_SOFTPLUS: dt holds the raw projection d; the step size is
 *                   softplus(d + dt_bias[h]) = log(1 + e^{d + dt_bias[h]}) > 0 (the step
 *                   is a positive projection of the token, Sec. 2 "Mamba-2 parameterisation").
 *   M3_LAM_SIGMOID: lam holds u; the trapezoid weight is sigma(u) = 1 / (1 + e^{-u})
 *                   (Appendix F, default parameterisation lambda_t = sigma(u_t)).
 * Positions past the end of the sequence are not tokens and stay zero.
 *   M3_DISC_ZOH:    the zero-order-hold discretisation of Mamba-1/2 instead of the
 *                   exponential-trapezoidal one ("Mamba-3：推理优先的状态空间模型", Sec. 1.2):
 *                   h_t = alpha_t h_{t-1} + gamma_t B_t x_t with gamma_t = (alpha_t - 1) / A_t
 *                   and no previous-token term; lam is not used. The rotation is unchanged. */
#define M3_DT_SOFTPLUS 1u
#define M3_LAM_SIGMOID 2u
#define M3_DISC_ZOH 4u
/* m3_scan_bwd only: compute every product of the backward in fp32 on the CUDA cores (the
 * sequential sweeps), also where the chunked tensor-core backward applies. Other entry points
 * ignore it. */
#define M3_BWD_FP32 8u

typedef struct {
    const void* x;        /* [b, L, H, R, P]   in_dtype                                   */
    const void* B;        /* [b, L, G, R, N]   in_dtype, raw (before norm and bias)       */
    const void* C;        /* [b, L, G, R, N]   in_dtype, raw                              */
    const void* theta;    /* [b, L, H, N/2]    in_dtype: per-step angle rate; the step's
                             rotation angle is dt * theta (Prop. 2)                     */
    const float* dt;      /* [b, L, H] step size, > 0 (raw projection with M3_DT_SOFTPLUS) */
    const float* A;       /* [b, L, H] decay rate, < 0                                     */
    const float* lam;     /* [b, L, H] trapezoid weight in [0, 1] (lam = 1: Euler), or the
                             raw u of sigma(u) with M3_LAM_SIGMOID                         */
    const float* B_bias;  /* [H, R, N] added after the norm, or NULL for zero              */
    const float* C_bias;  /* [H, R, N] or NULL                                             */
    const float* dt_bias; /* [H] added to dt before the softplus (M3_DT_SOFTPLUS only), or
                             NULL for zero                                                 */
} m3_inputs;

/* Recurrent state of every (batch, head) unit. Each unit owns its slice of every field. */
typedef struct {
    float* h;      /* [b, H, N, P] fp32, state in the rotated (RoPE) frame: prod R_s^T h  */
    float* phi;    /* [b, H, N/2]  fp32 cumulative angle sum_s dt_s theta_s               */
    void* prev_B;  /* [b, H, R, N] in_dtype: raw B of the last token seen (per head copy) */
    void* prev_x;  /* [b, H, R, P] in_dtype: x of the last token seen                     */
} m3_state;
/* The MIMO projections around one decode step (Appendix C). The step's input arrives as X'
 * and is expanded per rank in the kernel, X[r][p] = W_X[h][r][p] X'[p]; the output is gated
 * and contracted over the ranks, O'[p] = sum_r W_O[h][r][p] Y[r][p] SiLU(W_Z[h][r][p] Z'[p]),
 * with SiLU(z) = z / (1 + e^{-z}) and Y the SSM output of X. The paper's weights belong to the
 * layer (P x R); here every head has its own. */
typedef struct {
    const void* x_in;   /* [b, H, P] in_dtype: X' of the token                              */
    const void* z_in;   /* [b, H, P] in_dtype: Z' of the token                              */
    const float* W_X;   /* [H, R, P]                                                         */
    const float* W_Z;   /* [H, R, P]                                                         */
    const float* W_O;   /* [H, R, P]                                                         */
} m3_proj;

/* An all-zero state is the state of an empty sequence: h_{-1} = 0, x_{-1} = 0, so the first
 * step is h_0 = gamma_0 B_0 x_0 (Sec. 3.1.3). */

/* Bytes of device workspace m3_scan_fwd needs for these dims (>= 256), or 0 if the dims are
 * invalid or unsupported: a 256-byte status header, the per-token RMS scales of B and C, and
 * for few long sequences (which the scan cuts into segments that run in parallel) one fp32
 * state per sequence and segment. Depends on the current device's SM count. */
M3_API size_t m3_scan_workspace_bytes(const m3_dims* dims);

/* Chunked parallel prefill scan over a whole sequence (Sec. 3.1.3 parallel form, Sec. 3.3
 * chunked algorithm). The chunk length is a tile size: the result does not depend on it
 * beyond rounding. bf16 inputs with N = 128 and P = 64 run on the tensor cores when
 * chunk * R = 64 (any R) or chunk * R = 128 (R <= 4, a warp-specialised kernel with one CTA
 * per (batch, head) and per SM); other shapes, other chunk lengths and fp32 run on the
 * CUDA cores in exact fp32.
 *   init      state before token 0, or NULL for a fresh sequence (all zeros).
 *   final     where to write the state after token L-1, or NULL to skip; may alias init.
 *   y         [b, L, H, R, P] in_dtype output, y_t = H_t^T Cbar_t.
 *   workspace device buffer of at least m3_scan_workspace_bytes(dims) bytes, 256-byte
 *             aligned, its first 256 bytes (the status header) zero before its first use
 *             (e.g. one cudaMemsetAsync). A call that does not time out leaves the header
 *             zero, so the workspace is reused without resetting; the rest is scratch. Two
 *             calls that may run at the same time need separate workspaces.
 * Asynchronous: returns after launching. A device-side timeout (a wait between CTAs that
 * exceeded its bound) is reported by m3_scan_check after the stream has synchronised. */
M3_API m3_status m3_scan_fwd(const m3_dims* dims, const m3_inputs* in, const m3_state* init,
                      const m3_state* final_state, void* y, void* workspace,
                      size_t ws_bytes, void* stream);

/* One-token decode step: exactly one iteration of the recurrence for every unit, as
 * "Mamba-3: Improved Sequence Modeling using State Space Principles" states it for
 * inference: the trapezoidal update h_t = alpha_t h_{t-1} + beta_t Bbar_{t-1} x_{t-1}^T +
 * gamma_t Bbar_t x_t^T (Sec. 3.1.1 Prop. 1) with B and C rotated by the cumulative angle
 * carried in phi (Sec. 3.2.2 Prop. 4), then y_t = h_t^T Cbar_t; MIMO as in Appendix C
 * (H_t = a_t H_{t-1} + B_t X_t^T, Y_t = H_t^T C_t). prev_B and prev_x carry the token that
 * the beta term of the next step reads.
 *   dims->seqlen must be 1; `in` points at one token: x [b,1,H,R,P], B, C [b,1,G,R,N] ...
 *   state_in  the state before the token (required).
 *   state_out where to write the state after it; may be the same buffers as state_in.
 *   y         [b, H, R, P] in_dtype. */
M3_API m3_status m3_decode_step(const m3_dims* dims, const m3_inputs* in, const m3_state* state_in,
                         const m3_state* state_out, void* y, void* stream);

/* m3_decode_step with the MIMO projections fused (Appendix C, m3_proj): in->x is not read
 * (it may be NULL); the new state's prev_x is the expanded X, rounded to in_dtype; o
 * [b, H, P] in_dtype receives O'. All of proj's pointers are required, 16-byte aligned. */
M3_API m3_status m3_decode_step_proj(const m3_dims* dims, const m3_inputs* in,
                                     const m3_proj* proj, const m3_state* state_in,
                                     const m3_state* state_out, void* o, void* stream);

/* One segment's end state, for prefill split over devices along the sequence. */
typedef struct {
    float* h;        /* [b, H, N, P] fp32                                                    */
    float* phi;      /* [b, H, N/2]  fp32                                                    */
    float* lam_sum;  /* [b, H]       fp32: the segment's summed log-decay sum_t dt_t A_t     */
} m3_seg_state;

/* The recurrence over the tokens of `in` from `init`, without the output y: writes the state
 * after the last token (h and phi exactly as m3_scan_fwd's final state) and the summed
 * log-decay. For prefill split along the sequence over devices (context parallelism): each
 * device runs its own tokens, device 0 from the true initial state and every other one from
 * h = 0, phi = 0 with the previous device's last token as prev_B (per head) and prev_x; the
 * results are gathered (stacked over devices) and m3_state_combine gives each device the
 * state at its start, from which it runs m3_scan_fwd with that token as prev_B, prev_x.
 * The segments' contributions are exact by linearity (Sec. 3.1.1 Prop. 1) and the rotation
 * of the frame (Sec. 3.2.2 Prop. 4). Tensor-core shapes only (bf16, N = 128, P = 64,
 * chunk * R = 64), else M3_ERR_UNSUPPORTED. workspace: at least m3_scan_workspace_bytes. */
M3_API m3_status m3_scan_state(const m3_dims* dims, const m3_inputs* in, const m3_state* init,
                               const m3_seg_state* out, void* workspace, size_t ws_bytes,
                               void* stream);

/* The state after the last token of segment nseg-1 from the end states of segments
 * 0 .. nseg-1 stacked in seg (h [nseg, b, H, N, P], phi [nseg, b, H, N/2], lam_sum
 * [nseg, b, H]), run as m3_scan_state describes: h <- e^{lam_j} h + R(-phi_j) h_j with
 * phi_j the true angle at segment j's start. Writes h_out [b, H, N, P] and phi_out
 * [b, H, N/2]. Any supported N, P. */
M3_API m3_status m3_state_combine(const m3_dims* dims, int nseg, const m3_seg_state* seg,
                                  float* h_out, float* phi_out, void* stream);

/* ---- Backward pass of the prefill scan (the training side of the same recurrence) ----
 * Gradients of  L = sum(y * dy) + <final state, dfinal>  with respect to every input of
 * m3_scan_fwd and to its initial state, for the forward that m3_scan_fwd computes with the
 * same dims, inputs and init (Sec. 3.1.1 Prop. 1, Sec. 3.2.2 Prop. 4, Sec. 3.4, Appendix C;
 * the flags' transforms are differentiated too). All gradients are fp32. */
typedef struct {
    float* dx;        /* [b, L, H, R, P]                                                      */
    float* dB;        /* [b, L, G, R, N] with respect to the raw B (heads of a group summed)  */
    float* dC;        /* [b, L, G, R, N]                                                      */
    float* dtheta;    /* [b, L, H, N/2]                                                       */
    float* ddt;       /* [b, L, H] with respect to dt as passed (the raw projection under
                         M3_DT_SOFTPLUS)                                                     */
    float* dA;        /* [b, L, H]                                                            */
    float* dlam;      /* [b, L, H] with respect to lam as passed (u under M3_LAM_SIGMOID; zero
                         under M3_DISC_ZOH, which does not use it)                           */
    float* dB_bias;   /* [H, R, N], or NULL to skip                                           */
    float* dC_bias;   /* [H, R, N], or NULL                                                   */
    float* ddt_bias;  /* [H], or NULL; zero unless M3_DT_SOFTPLUS                             */
} m3_grads;

/* Gradient with respect to a state (all fp32, shapes as m3_state). As an input a NULL field
 * (or a NULL struct) is zero; as an output a NULL field is not written. */
typedef struct {
    float* h;       /* [b, H, N, P] */
    float* phi;     /* [b, H, N/2]  */
    float* prev_B;  /* [b, H, R, N] with respect to the raw previous B */
    float* prev_x;  /* [b, H, R, P] */
} m3_state_grad;

/* Workspace bytes m3_scan_bwd needs (0 for invalid dims): a 256-byte status header, two
 * fp32 [b, L, H, R, N] buffers plus O(b H (L + N L / 16)) floats, and where the chunked
 * tensor-core form runs (see m3_scan_bwd) 16 KB per unit and 64-token chunk for the chunk
 * states plus O(b H N P) floats. Any content: the call resets the status word itself. */
M3_API size_t m3_scan_bwd_workspace_bytes(const m3_dims* dims);

/* Gradients of the prefill scan ("Mamba-3: Improved Sequence Modeling using State Space
 * Principles", the recurrence of Sec. 3.1.1 Prop. 1 with the rotation of Sec. 3.2.2 Prop. 4,
 * differentiated; Sec. 3.3 for the chunked form).
 * dims, in, init: as given to m3_scan_fwd (dims->chunk is not used here). dy [b, L, H, R, P]
 * in_dtype. dfinal: the final state's gradient, or NULL. grads: dx .. dlam are required
 * (16-byte aligned) and overwritten; the bias gradients are overwritten when not NULL.
 * dinit: where to write the initial state's gradient, or NULL. workspace: 256-byte aligned,
 * at least m3_scan_bwd_workspace_bytes. Any supported N, P, R, dtype and flags; asynchronous
 * on `stream`.
 * Two forms compute the same gradients:
 *  - bf16 inputs with R in {1, 2, 4, 8}, N = 128, P = 64 and H a multiple of 4 run the
 *    chunked form on the tensor cores (chunks of 64 (token, rank) rows, bf16 operands with
 *    fp32 accumulators, fp32 state adjoint), bitwise reproducible run to run. Its bounded
 *    waits report a timeout through the workspace's status word, which m3_scan_check reads
 *    after the stream has synchronised.
 *  - every other shape, and any shape with M3_BWD_FP32 in dims->flags, runs two sequential
 *    sweeps in fp32 on the CUDA cores; not bitwise reproducible run to run (some sums use
 *    atomic adds, whose order varies in the last bits). */
M3_API m3_status m3_scan_bwd(const m3_dims* dims, const m3_inputs* in, const m3_state* init,
                             const void* dy, const m3_state_grad* dfinal,
                             const m3_grads* grads, const m3_state_grad* dinit,
                             void* workspace, size_t ws_bytes, void* stream);

/* After the stream that ran m3_scan_fwd (or m3_scan_bwd, on its workspace) has synchronised:
 * M3_OK, or M3_ERR_TIMEOUT if a
 * bounded inter-CTA wait gave up (the outputs of that call are then incomplete). Performs
 * one blocking 4-byte device-to-host copy; after a timeout it also re-zeroes the workspace
 * header (blocking) so the workspace can be reused. */
M3_API m3_status m3_scan_check(void* workspace);

/* m3_scan_fwd for callers that cannot allocate device memory when they run the scan: a
 * serving runtime that fixes all of its device memory before it starts and allows no
 * allocation afterwards, code running in a step whose memory was planned in advance, or an
 * embedding with no allocator to hand out. It is m3_scan_fwd without the workspace argument;
 * the pages define no counterpart, it exists only for those callers.
 *   Scratch: a 1 MiB array that is part of the library (a __device__ variable, so every GPU
 *   that loads the library keeps its own copy until the process exits). The call itself
 *   allocates and frees nothing; the caller still passes inputs, state and y as above.
 *   First call on a device: looks up the array's device address (cudaGetSymbolAddress) with
 *   that device current and caches it, so make the first call on each device before any
 *   stream capture.
 *   Sharing: all calls on a device use the same array, and it keeps what the last call left
 *   (each call clears the status bytes it needs at zero first). Calls whose work can overlap
 *   on the GPU (different streams, or different host threads) race on the array: serialise
 *   them, or use m3_scan_fwd with one workspace each.
 *   Limit: dims whose scan cannot run in 1 MiB return M3_ERR_UNSUPPORTED. With BC
 *   normalisation on, the tensor-core paths keep 8 bytes of RMS scales per row and the
 *   array holds 131040 rows (1 MiB less a 256-byte status header), so the call runs when
 *   batch * ceil(seqlen / chunk) * chunk * ngroups * rank <= 131040 (seqlen padded up to
 *   whole chunks) and is rejected above that. With BC normalisation off, or on the fp32
 *   path, there is no such limit. Few long sequences, which m3_scan_fwd cuts into parallel segments, use only
 *   as many segments as the rest of the array holds the end states of (possibly one): the
 *   results are the same, the time may be longer. A device-side wait that gives up cannot
 *   be reported here; use m3_scan_fwd and m3_scan_check when that matters. */
M3_API m3_status m3_scan_fwd_noalloc(const m3_dims* dims, const m3_inputs* in,
                                     const m3_state* init, const m3_state* final_state,
                                     void* y, void* stream);

/* Static description of a status code. */
M3_API const char* m3_status_str(m3_status s);

/* Human-readable reason for the most recent failed call on this thread ("" if none). */
M3_API const char* m3_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* M3_H_ */
