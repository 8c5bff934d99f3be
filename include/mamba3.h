/*
 * mamba3.h -- C ABI of the Mamba-3 selective-recurrence library (sm_100a).
 *
 * The layer's core computation, per (batch b, head h), token t = 1..L:
 *
 *   h_t = alpha_t h_{t-1} + beta_t B~_{t-1}^T x_{t-1} + gamma_t B~_t^T x_t
 *   y_t = C~_t h_t + D_h x_t
 *   alpha_t = exp(dt_t A_h),  beta_t = (1 - lam_t) dt_t alpha_t,  gamma_t = lam_t dt_t
 *
 * Sources (pages on the Mamba-3 paper, "Mamba-3: 2x smaller state ..." by
 * MarkTechPost, Korean translation):
 *   section 1.1  exponential-trapezoidal discretisation: the three-term update;
 *   section 1.2  complex state via the RoPE trick: B~, C~ are B, C with each
 *                adjacent pair (2k, 2k+1) rotated by -Phi_t,k where
 *                Phi_t = Phi_0 + sum_{s<=t} dt_s theta_s (the angle accumulated
 *                over time steps);
 *   section 1.3  MIMO: B_t is N x R and x_t is P x R; B~_t^T x_t means
 *                sum_r B~_t[r]^T x_t[r] and y_t has one P-vector per rank.
 * The readout C~_t h_t + D x_t is the standard SSM readout (not printed on
 * the pages).  A is one real scalar per head.
 *
 * Conventions (all entry points):
 *  - Every pointer is a DEVICE pointer unless stated otherwise, owned by the
 *    caller.  The library never allocates, frees or synchronises (except
 *    mamba3_device_status, which synchronises the stream it is given); work
 *    is enqueued on `stream` (a cudaStream_t passed as void*, NULL = legacy
 *    default stream).
 *  - Layouts are dense row-major with the last index fastest:
 *      x, y      [batch, seqlen, nheads, rank, headdim]      (in_dtype)
 *      B, C      [batch, seqlen, G, rank, dstate]            (in_dtype)
 *                G = dims->ngroups (nheads when 0): the pages give each head
 *                its own B and C; sharing them among G groups of consecutive
 *                heads is the Mamba line's grouped form (head h reads row
 *                h / (nheads / G)).
 *      theta     [batch, seqlen, nheads, dstate/2]           (in_dtype)
 *      dt, lam   [batch, seqlen, nheads]                     (in_dtype)
 *      A, D      [nheads]                                    (float32)
 *    For the decode step drop the seqlen axis.
 *  - Every input and output pointer must be 16-byte aligned.
 *  - Host-detectable errors return a negative status before anything is
 *    enqueued.  No C++ exception crosses the ABI.  There is no CPU fallback:
 *    without a CUDA device the calls return MAMBA3_ERR_CUDA.
 */
#ifndef MAMBA3_H
#define MAMBA3_H

#include <stddef.h>

#if defined(__GNUC__)
#define MAMBA3_API __attribute__((visibility("default")))
#else
#define MAMBA3_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MAMBA3_OK = 0,
  MAMBA3_ERR_INVALID = -1,     /* null pointer, bad size, misaligned pointer */
  MAMBA3_ERR_UNSUPPORTED = -2, /* valid arguments outside the compiled shapes */
  MAMBA3_ERR_WORKSPACE = -3,   /* workspace missing or smaller than required */
  MAMBA3_ERR_CUDA = -4,        /* a CUDA runtime/driver call or launch failed */
  MAMBA3_ERR_TIMEOUT = -5      /* a bounded on-device wait gave up (device status) */
} mamba3_status;

typedef enum { MAMBA3_F32 = 0, MAMBA3_BF16 = 1 } mamba3_dtype;

typedef struct {
  int batch;    /* b >= 1 */
  int seqlen;   /* L >= 0 (ignored by mamba3_decode_step) */
  int nheads;   /* H >= 1 */
  int headdim;  /* P: multiple of 4 */
  int dstate;   /* N: even */
  int rank;     /* R: 1 (SISO) or 2, 4, 8 (MIMO) */
  int chunk;    /* Q tokens per chunk for the prefill; 0 = library default */
  mamba3_dtype in_dtype; /* dtype of x, B, C, theta, dt, lam and y */
  int ngroups;  /* G rows of B and C per token: 0 = one per head (G = nheads);
                 * otherwise G divides nheads and heads g*(H/G) .. (g+1)*(H/G)-1
                 * share row g.  Added in ABI 2.00. */
} mamba3_dims;

/*
 * Recurrent state of one layer (float32, device memory, caller-owned).
 * It is what a decode step continues from and what a prefill exports:
 *   h      [batch, nheads, dstate, headdim]  state in the frame rotated by -Phi
 *                                            (row 2k = real, 2k+1 = imaginary part)
 *   b_prev [batch, nheads, rank, dstate]     B~ of the last token (already rotated)
 *   x_prev [batch, nheads, rank, headdim]    x of the last token
 *   angle  [batch, nheads, dstate/2]         Phi of the last token, wrapped to [-pi, pi)
 * A zero state (h = 0, b_prev = 0, x_prev = 0, angle = 0) is the start of a sequence.
 */
typedef struct {
  float* h;
  float* b_prev;
  float* x_prev;
  float* angle;
} mamba3_state;

/* Bytes of device workspace mamba3_scan_fwd needs for `dims` (>= 256; the
 * first 256 bytes hold the device status word).  Returns 0 for invalid dims. */
MAMBA3_API size_t mamba3_scan_workspace_bytes(const mamba3_dims* dims);

/*
 * Chunked prefill over a whole sequence (sections 1.1-1.3 above).
 *   init         nullable: NULL = zero state; otherwise all four fields non-null.
 *   D            nullable: NULL = no skip term.
 *   final_state  nullable: NULL = do not export; otherwise all four fields
 *                non-null.  It may alias `init` (in-place continuation).
 *   workspace    device memory of at least mamba3_scan_workspace_bytes(dims);
 *                its status word is reset by this call and read back with
 *                mamba3_device_status.  With mamba3_scan_fwd_workspace_bytes(dims)
 *                the call also runs its long-sequence segments or its split
 *                last wave (declared below), which give the same y and state.
 *                A workspace serves one call at a time: calls that overlap on
 *                the GPU need workspaces of their own (a split launch that
 *                draws a ticket past its range, which only a shared workspace
 *                causes, computes nothing and reports MAMBA3_ERR_TIMEOUT).
 * Numerics: float32 arithmetic and state; bf16 inputs feed bf16 tensor-core
 * products with float32 accumulation.  y is written in in_dtype.
 */
MAMBA3_API int mamba3_scan_fwd(const mamba3_dims* dims, const void* x, const void* B, const void* C,
                    const void* theta, const void* dt, const void* lam, const float* A,
                    const float* D, const mamba3_state* init, void* y,
                    const mamba3_state* final_state, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * The prefill from host buffers (mamba3_scan_fwd with x, B, C, theta, dt, lam and
 * y in host memory; page-locked memory lets the copies run asynchronously).  The
 * batch is cut into up to 8 sub-batches that cycle through two slots of `stage`:
 * while sub-batch i is computed on `stream`, the inputs of sub-batch i + 1 are
 * copied in and y of sub-batch i - 1 is copied out on two streams of the call's
 * own, so that both copy directions and the kernels overlap.  Every batch row is
 * an independent set of (b, h) units, so the result equals mamba3_scan_fwd's.
 *   A, D, init, final_state   device memory, as for mamba3_scan_fwd.
 *   stage        device memory of at least mamba3_scan_fwd_host_stage_bytes(dims)
 *                (16-byte aligned); its first 256 bytes are the status word
 *                (mamba3_device_status), reset by this call.
 *   stream       the call's work, including the last copy of y into host memory,
 *                is ordered on `stream`: synchronising it makes y readable.
 * Errors are reported before anything is enqueued, except MAMBA3_ERR_CUDA.
 * Host arrays are read and y written asynchronously: they must stay valid and
 * unmodified until `stream` has passed this call.  Section 1.1-1.3 as above.
 */
MAMBA3_API size_t mamba3_scan_fwd_host_stage_bytes(const mamba3_dims* dims);
MAMBA3_API int mamba3_scan_fwd_host(const mamba3_dims* dims, const void* x, const void* B, const void* C,
                                    const void* theta, const void* dt, const void* lam, const float* A,
                                    const float* D, const mamba3_state* init, void* y,
                                    const mamba3_state* final_state, void* stage, size_t stage_bytes,
                                    void* stream);

/*
 * One decode step for every (batch, head), in place on `state`
 * (section 1.3: the state is streamed once; the rank-R update and readout
 * happen in registers).  Per-token inputs have no seqlen axis:
 *   x [b,H,R,P], B/C [b,H,R,N], theta [b,H,N/2], dt/lam [b,H]; y [b,H,R,P].
 * D nullable.  dims->seqlen and dims->chunk are ignored.
 */
MAMBA3_API int mamba3_decode_step(const mamba3_dims* dims, const mamba3_state* state, const void* x,
                       const void* B, const void* C, const void* theta, const void* dt,
                       const void* lam, const float* A, const float* D, void* y, void* stream);

/*
 * Fused B/C normalisation ahead of the recurrence ("Mamba-3: 2x smaller state
 * ..." (MarkTechPost, Korean translation), section 2: RMS norm of B and C and a
 * head-specific bias).  For every (b, t, h, r) row of the raw projections,
 *     B[n] = B_raw[n] / sqrt(mean_n B_raw^2 + eps) * w_B[h,r,n] + bias_B[h,r,n]
 * (C likewise), computed in float32 from the raw inputs and then rotated as in
 * mamba3_scan_fwd.  w_B, w_C, bias_B, bias_C: device float32 [H, R, N],
 * contiguous, 4-byte aligned, each nullable (weight 1, bias 0); eps >= 0.
 */
typedef struct {
  const float *w_B, *w_C, *bias_B, *bias_C;
  float eps;
} mamba3_bc_norm;

/*
 * mamba3_scan_fwd with raw B and C projections (layouts as B and C there) and
 * the normalisation `norm` (not nullable) fused in front of the rotation.  The
 * exported state (b_prev) holds the normalised, rotated B, so a continuation
 * may use either entry point.  Supported: bf16 inputs, P = 64, N in {64, 128},
 * R in {1, 2, 4} (the tensor-core path); other shapes return
 * MAMBA3_ERR_UNSUPPORTED before anything is enqueued.
 */
MAMBA3_API int mamba3_scan_fwd_bcnorm(const mamba3_dims* dims, const void* x, const void* B_raw,
                                      const void* C_raw, const void* theta, const void* dt, const void* lam,
                                      const float* A, const float* D, const mamba3_bc_norm* norm,
                                      const mamba3_state* init, void* y, const mamba3_state* final_state,
                                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * mamba3_decode_step with raw B and C of the token and the normalisation
 * `norm` (not nullable) fused in front of the rotation.  Supported: P = 64,
 * N in {64, 128}, R in {1, 2, 4}, 16-byte aligned state and input pointers;
 * other cases return MAMBA3_ERR_UNSUPPORTED.
 */
MAMBA3_API int mamba3_decode_step_bcnorm(const mamba3_dims* dims, const mamba3_state* state, const void* x,
                                         const void* B_raw, const void* C_raw, const void* theta, const void* dt,
                                         const void* lam, const float* A, const float* D,
                                         const mamba3_bc_norm* norm, void* y, void* stream);

/*
 * Time-varying decay ("Mamba-3: 2x smaller state ..." (MarkTechPost, Korean
 * translation), section 1.1 writes the discretisation with a per-step A_t):
 * mamba3_scan_fwd / mamba3_decode_step with the per-head A replaced by a rate
 * per token and head, A_t, so that alpha_t = exp(dt_t A_t) and
 * beta_t = (1 - lam_t) dt_t alpha_t.  A_t has the dtype of x and the layout of
 * dt: [b, L, H] for the prefill, [b, H] for the decode step; not nullable.
 * Every other argument, layout and result is that of the plain entry point.
 */
MAMBA3_API int mamba3_scan_fwd_at(const mamba3_dims* dims, const void* x, const void* B, const void* C,
                                  const void* theta, const void* dt, const void* lam, const void* A_t,
                                  const float* D, const mamba3_state* init, void* y,
                                  const mamba3_state* final_state, void* workspace, size_t workspace_bytes,
                                  void* stream);
MAMBA3_API int mamba3_decode_step_at(const mamba3_dims* dims, const mamba3_state* state, const void* x,
                                     const void* B, const void* C, const void* theta, const void* dt,
                                     const void* lam, const void* A_t, const float* D, void* y, void* stream);

/*
 * Backward pass of mamba3_scan_fwd: the gradients of a loss L given dL/dy and,
 * optionally, dL/d(exported state).  The pages give no gradient formulas; these
 * are the chain rule applied to the recurrence above (section 1.1), its
 * rotation (section 1.2) and the rank-R products (section 1.3), in reverse
 * order over the sequence.
 *   x .. D, init  as for mamba3_scan_fwd (A per head; B, C per head or grouped
 *                 by dims->ngroups, dB, dC then summed over each group's heads;
 *                 dims->chunk is ignored).
 *   dy            layout and dtype of y.
 *   d_final       nullable: float32 gradients of the four exported state fields
 *                 (all non-null when given).
 *   dx, dB, dC, dtheta, ddt, dlam
 *                 outputs, the layouts and dtype of x, B, C, theta, dt, lam.
 *   dA, dD        outputs, float32 [nheads], summed over batch and tokens;
 *                 overwritten (zeroed on `stream`, then accumulated).  dD nullable.
 *   d_init        nullable: float32 gradients of the four initial-state fields
 *                 (with init NULL, those of a zero initial state).
 *   workspace     at least mamba3_scan_bwd_workspace_bytes(dims), after the
 *                 256-byte status word: the state at every chunk start, kept
 *                 between the forward state march and the reverse sweep.
 *                 Tensor-core path (bf16, P = 64, N in {64, 128}, R in {1, 2, 4},
 *                 seqlen >= 1): per (b, h) and 64-row chunk (Q = 64 / rank tokens)
 *                 a bf16 N x P tile and N/2 float angles, i.e.
 *                 batch * nheads * ceil(seqlen / Q) * (128 N + 2 N) bytes (SISO
 *                 b8 L2048 H64 N128: 272 MB); with grouped B/C then the fp32 sums
 *                 of dB and dC, 2 * batch * seqlen * ngroups * rank * dstate
 *                 floats.  Other shapes (SIMT path): per (b, h) and chunk of
 *                 Q = 32 / rank tokens, N P + N/2 floats; with grouped B/C then
 *                 the same fp32 group sums (2 * batch * seqlen * ngroups * rank *
 *                 dstate floats; each head adds its share with atomics).
 *                 With more (b, h) units than the 148 SMs the tensor-core path
 *                 also splits the last wave of its reverse sweep (as the prefill
 *                 does, see mamba3_scan_fwd_workspace_bytes): the CTA that sweeps
 *                 a unit's end hands the adjoint of the carried state, the running
 *                 angle-gradient sum and one token's pending dt, lam gradient share
 *                 over to the CTA that sweeps its start; mamba3_scan_bwd_workspace_bytes
 *                 includes that region (256 bytes, then k + 1 counters rounded up to
 *                 256 bytes and k (N P + N/2 + 4) floats), and a workspace of the
 *                 size above without it runs unsplit.
 * Products on the tensor cores take bf16 operands with float32 accumulation;
 * everything else is float32.  Returns MAMBA3_ERR_UNSUPPORTED for N, P whose
 * per-chunk tiles exceed shared memory.
 * mamba3_scan_bwd_at is the same for mamba3_scan_fwd_at: A_t [b, L, H] (dtype of x)
 * in place of A, and dA_t (layout and dtype of A_t, not nullable) in place of dA.
 */
MAMBA3_API size_t mamba3_scan_bwd_workspace_bytes(const mamba3_dims* dims);
MAMBA3_API int mamba3_scan_bwd(const mamba3_dims* dims, const void* x, const void* B, const void* C,
                               const void* theta, const void* dt, const void* lam, const float* A,
                               const float* D, const mamba3_state* init, const void* dy,
                               const mamba3_state* d_final, void* dx, void* dB, void* dC, void* dtheta,
                               void* ddt, void* dlam, float* dA, float* dD, const mamba3_state* d_init,
                               void* workspace, size_t workspace_bytes, void* stream);
MAMBA3_API int mamba3_scan_bwd_at(const mamba3_dims* dims, const void* x, const void* B, const void* C,
                                  const void* theta, const void* dt, const void* lam, const void* A_t,
                                  const float* D, const mamba3_state* init, const void* dy,
                                  const mamba3_state* d_final, void* dx, void* dB, void* dC, void* dtheta,
                                  void* ddt, void* dlam, void* dA_t, float* dD, const mamba3_state* d_init,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * Output side of the layer: the pre-gate grouped RMS norm and the gate
 * ("Mamba-3: 2x smaller state ..." (MarkTechPost, Korean translation),
 * section 2: a grouped RMS norm ahead of the output gate in hybrids).  Per token
 * and norm group g of nheads / groups consecutive heads, over the group's
 * channels c = (h, r, p):
 *     out[c] = y[c] / sqrt(mean_c y[c]^2 + eps) * w[h, r, p] * silu(z[c]),
 * silu(z) = z / (1 + e^{-z}) (the pages do not name the gate's nonlinearity;
 * this is the Mamba line's).  An all-zero group with eps = 0 gives 0.
 *   dims   batch, seqlen (1 for one decode step's output), nheads, headdim, rank,
 *          in_dtype; dstate, chunk and ngroups are ignored.
 *   y, z, out  [batch, seqlen, nheads, rank, headdim] in_dtype, 16-byte aligned;
 *          out may alias y.
 *   w      float32 [nheads, rank, headdim], 16-byte aligned, or NULL (weight 1).
 *   groups divides nheads (nheads: one group per head); eps >= 0.
 * HBM-bound: y and z read once, out written once; computed in float32.
 */
MAMBA3_API int mamba3_gated_norm(const mamba3_dims* dims, int groups, const void* y, const void* z, const float* w,
                                 float eps, void* out, void* stream);

/*
 * Workspace with which mamba3_scan_fwd (and its _at variant) runs a long
 * sequence over few (batch, head) units in segments: with fewer units than the
 * GPU has SMs, the sequence is cut into S segments (S divides seqlen, at least
 * 1024 tokens each), every segment's end state from a zero state is computed,
 * the segment states are chained in order (a decay, a rotation by the entering
 * angle and the sum, exact up to rounding), and the prefill runs on the b S
 * segments at once.  The constant-size state and the angle summed over time
 * steps ("Mamba-3 paper review" (no1joon.github.io), Table 7 discussion;
 * "Mamba-3: 2x smaller state ..." (MarkTechPost, Korean translation), section
 * 1.2) make the split exact.  Returns the status word's 256 bytes plus
 * 2 b S H (N P + R N + R P + N/2) floats, or 256 when `dims` do not qualify
 * (bf16, P = 64, N in {64, 128}, R in {1, 2, 4}, seqlen >= 2048, b H < 148);
 * 0 for invalid dims.  Any workspace of at least mamba3_scan_workspace_bytes
 * is accepted: a smaller one than this runs the sequence unsegmented.
 */
MAMBA3_API size_t mamba3_scan_segmented_workspace_bytes(const mamba3_dims* dims);

/*
 * For testing the segmented prefill on small problems only: while S >= 2, the
 * prefill (and mamba3_scan_segmented_workspace_bytes) uses S segments whenever S
 * divides seqlen and the shape has the segmented path, whatever the sequence
 * length and unit count; 0 restores the library's own choice.  Process-wide.
 */
MAMBA3_API int mamba3_test_set_segments(int S);

/*
 * The workspace with which mamba3_scan_fwd (and its _at and _bcnorm forms) runs
 * its best schedule for `dims`: the segmented prefill where that applies (then
 * equal to mamba3_scan_segmented_workspace_bytes), otherwise the status block
 * plus what the tensor-core prefill needs to split its last wave.  With U = b H
 * units on the 148 SMs, the last of ceil(U / 148) waves of one CTA per unit holds
 * only U mod 148 units; the library instead runs k units in two CTAs, chunks
 * [0, c1) in the first wave and [c1, n) in the last, the second continuing from
 * the carried state and the accumulated angle that the first hands over in the
 * workspace (the chunk recurrence of "Mamba-3: 2x smaller state ..." (MarkTechPost,
 * Korean translation), sections 1.1-1.2, crosses a chunk boundary the same way
 * inside one CTA, so y and the final state are those of the unsplit prefill bit
 * for bit).  The space is 256 bytes of status, k 4-byte flags rounded up to 256
 * bytes, and k (N P + N/2) floats, k < 148 + 32; 256 when the shape gains nothing
 * from a split (U a multiple of 148, U <= 148, or no tensor-core path).  0 for
 * invalid dims.  Any workspace of at least mamba3_scan_workspace_bytes works: a
 * smaller one than this runs without the split.
 */
MAMBA3_API size_t mamba3_scan_fwd_workspace_bytes(const mamba3_dims* dims);

/*
 * For testing the split last wave only: k > 0 splits units 0 .. k-1 after c1
 * chunks whenever k <= b H and 1 <= c1 < the number of chunks (otherwise no
 * split); k < 0 never splits; k = 0 restores the library's plan.  Returns
 * MAMBA3_ERR_INVALID for k > 0 with c1 < 1.  Process-wide.
 */
MAMBA3_API int mamba3_test_set_split(int k, int c1);

/* Synchronises `stream`, then returns the device status word that the last
 * mamba3_scan_fwd on `workspace` left (MAMBA3_OK or MAMBA3_ERR_TIMEOUT), or
 * MAMBA3_ERR_CUDA / MAMBA3_ERR_INVALID. */
MAMBA3_API int mamba3_device_status(const void* workspace, void* stream);

/*
 * MIMO rank-R projections around the recurrence ("Mamba-3: 2x smaller state
 * ..." (MarkTechPost, Korean translation), section 1.3: MIMO raises the rank of
 * the input and output projections so that x_t is P x R).  The page prints no
 * weights; the reading here is one dense matrix per head on each side:
 *   up:   x[t, h, r, p] = sum_q Wx[h, r P + p, q] u[t, h, q]
 *   down: o[t, h, p]    = sum_{r, q} Wy[h, p, r P + q] y[t, h, r, q]
 * over every (batch, token) pair t.  With z non-null the down projection is
 * followed by the output side of section 2 for norm groups of one head:
 *   out = o / sqrt(mean_p o^2 + eps) * w[h, p] * silu(z[t, h, p])
 * (w nullable: weight 1; an all-zero row with eps = 0 gives 0).
 *   dims   batch, seqlen, nheads, headdim (P), rank (R), in_dtype; dstate,
 *          chunk and ngroups are ignored.
 *   u [b, L, H, P]; Wx [H, R P, P]; x [b, L, H, R, P]        (bf16)
 *   y [b, L, H, R, P]; Wy [H, P, R P]; z, out [b, L, H, P]   (bf16); w float32 [H, P]
 * Supported: bf16, P = 64, R in {1, 2, 4} (tcgen05 products per 128-token tile,
 * fp32 accumulation); other valid shapes return MAMBA3_ERR_UNSUPPORTED.  Every
 * pointer 16-byte aligned (w: 4).  Asynchronous on `stream`; no workspace (a
 * timed-out wait is reported by mamba3_library_status).
 */
MAMBA3_API int mamba3_mimo_up(const mamba3_dims* dims, const void* u, const void* Wx, void* x, void* stream);
MAMBA3_API int mamba3_mimo_down(const mamba3_dims* dims, const void* y, const void* Wy, const void* z,
                                const float* w, float eps, void* out, void* stream);

/*
 * Device status of the entry points that take no workspace (the decode steps
 * and the MIMO projections): their status words are library-owned, one per
 * device.  A kernel whose bounded wait for its own copies gives up records
 * MAMBA3_ERR_TIMEOUT there (and lets what it issued land before it exits).
 * The words are sticky: this call synchronises `stream`, returns the first code
 * recorded on the current device since the last call (MAMBA3_OK if none) and
 * clears them.  Shared by every such call on the device.
 */
MAMBA3_API int mamba3_library_status(void* stream);

/*
 * Bound of every on-device wait (the prefill's pipeline barriers, the decode
 * step's copy barriers, the backward pass's), in SM clock cycles; default
 * 4e9 (about 2 s).  A wait that reaches it ends its kernel with
 * MAMBA3_ERR_TIMEOUT in the status word; the kernel first lets every copy and
 * tensor-core operation it issued complete, so the context stays usable.
 * Process-wide, read at each launch; cycles >= 1000, else MAMBA3_ERR_INVALID.
 */
MAMBA3_API int mamba3_set_wait_limit(long long cycles);

/*
 * For testing the timeout path only: while `on` is non-zero, the prefill's
 * producer and the decode step issue none of their input copies, so every
 * kernel launched meanwhile ends with MAMBA3_ERR_TIMEOUT after the wait limit
 * (its outputs are then undefined).  Process-wide; off by default.
 */
MAMBA3_API int mamba3_test_withhold_loads(int on);

/*
 * Bytes of library-owned device scratch behind mamba3_scan_fwd_noalloc
 * (a file-scope device array; every GPU that loads the library holds it
 * until the process exits).
 */
#define MAMBA3_NOALLOC_SCRATCH_BYTES (1u << 20)

/*
 * mamba3_scan_fwd without a workspace argument.  The pages on the method have
 * no counterpart for this entry point; it exists for callers that cannot call
 * cudaMalloc themselves: code embedded in a host framework that owns all device
 * memory through its own pool (an allocation outside the pool can fail against
 * the pool's reservation), latency-critical serving loops (cudaMalloc/cudaFree
 * may synchronise the device and stall other streams), and runtimes that fix
 * their memory budget at start-up.
 *
 * Arguments, layouts and results are those of mamba3_scan_fwd; the scratch is
 * MAMBA3_NOALLOC_SCRATCH_BYTES of library-owned device memory instead of a
 * caller workspace.  Nothing is allocated and nothing is freed.
 *  - The first call on a device (with that device current) looks the scratch's
 *    device address up once (cudaGetSymbolAddress); make that first call
 *    before any stream capture on that device.  The address is kept for the
 *    life of the process: it assumes the device's primary context is never
 *    torn down (no cudaDeviceReset between calls).
 *  - Problems that need more scratch than MAMBA3_NOALLOC_SCRATCH_BYTES
 *    (mamba3_scan_workspace_bytes) are rejected with MAMBA3_ERR_WORKSPACE
 *    before anything is enqueued.
 *  - Every call on a device shares the same scratch and it keeps the last
 *    call's contents; the parts that must start at zero (the device status
 *    word) are cleared by each call on its stream.  Calls that overlap on the
 *    GPU (different streams without ordering between them) race on it.  For
 *    that reason this entry point never splits the last wave (see
 *    mamba3_scan_fwd_workspace_bytes).
 *  - The device status word stays in the library's scratch: use
 *    mamba3_scan_fwd with a caller workspace when mamba3_device_status is needed.
 */
MAMBA3_API int mamba3_scan_fwd_noalloc(const mamba3_dims* dims, const void* x, const void* B, const void* C,
                                       const void* theta, const void* dt, const void* lam, const float* A,
                                       const float* D, const mamba3_state* init, void* y,
                                       const mamba3_state* final_state, void* stream);

/* Static, human-readable text for a status code. */
MAMBA3_API const char* mamba3_status_string(int status);

/* Library ABI version (major * 100 + minor). */
MAMBA3_API int mamba3_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MAMBA3_H */
