/*
 * eot.h -- C ABI of libeot, blockwise band-support balanced log-domain Sinkhorn attention
 * for NVIDIA B200 (sm_100a).
 *
 * Method: "Blockwise Differentiable Sinkhorn Attention", technical summary (gist.science,
 * paper 2605.08123).  Per (batch, head) unit, with S_ij = scale <q_i, k_j> (the entropic
 * temperature absorbed into S, §2.1) on the fixed band support
 *     Omega = { (i, j) : i, j active, |i - j| <= W / 2 }          (§2.1; W / 2 rounds down)
 * and uniform marginals a = b over the active tokens, the forward pass runs
 *     T stopped balanced Sinkhorn steps from v = 0                (§2.1, stopped base)
 *         u_i = log a_i - LSE_{j : (i,j) in Omega} (S_ij + v_j)
 *         v_j = log b_j - LSE_{i : (i,j) in Omega} (S_ij + u_i)
 *     R more steps from (u0, v0), the differentiable tail          (§2.1, refinement tail)
 *     O = diag(1/a) P V,  P = exp(S + u(R) + v(R)) on Omega
 * and the backward pass is the exact adjoint of that tail w.r.t. Q, K, V with the base held
 * fixed (§2.2), computed from one reference plan P(R,R) per tile plus per-row and per-column
 * factors exp(u(k) - u(R)), exp(v(k) - v(R)) (the scaling-orbit identity of §2.2).
 * With the dustbin flag (§2.3) a dustbin token at ``dustbin_index`` is linked to every
 * active real token in both directions (and to itself when ``dustbin_self``); it carries
 * marginal ``dustbin_mass`` and the real tokens share 1 - dustbin_mass.  Positions after the
 * dustbin are inactive fillers.
 *
 * Conventions common to every call
 *   - All tensors are caller-owned device buffers, contiguous, [B, H, L, d] row-major for
 *     Q, K, V, O, dO, dQ, dK, dV (element type given by ``dtype``), [B, H, R+1, L] float32
 *     for the tail potentials, [B, L] uint8 for the mask.
 *   - The library never allocates device memory (all scratch lives in the caller's
 *     workspace) and keeps no global device state.
 *   - Calls are asynchronous and stream-ordered on ``stream`` (a cudaStream_t; NULL is the
 *     legacy default stream).  No host synchronisation happens inside fwd/bwd.
 *   - Argument errors are detected on the host before anything is enqueued; nothing is then
 *     launched and the status says why.  Launch failures return EOT_ERR_CUDA.
 *   - Conditions found on the device (a non-finite potential, a wait that ran out) set bits
 *     in a status word inside the workspace; read them with eot_last_device_status.  The
 *     kernels never trap.
 *   - B * H * L == 0 is an empty problem: the call validates and returns EOT_OK at once.
 *   - Rows of inactive tokens are written as 0 in O, dQ, dK, dV; their u and v are 0.
 */
#ifndef EOT_H_
#define EOT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define EOT_ABI_VERSION 1

typedef enum {
    EOT_OK = 0,
    EOT_ERR_INVALID_ARGUMENT = 1,   /* bad size, pointer or flag; nothing was launched */
    EOT_ERR_UNSUPPORTED = 2,        /* valid problem this library cannot run (e.g. impl/dtype) */
    EOT_ERR_WORKSPACE_TOO_SMALL = 3,
    EOT_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed */
    EOT_ERR_NONFINITE = 5,          /* device status: a non-finite potential was produced */
    EOT_ERR_TIMEOUT = 6             /* device status: a bounded wait inside a kernel ran out */
} eot_status;

typedef enum { EOT_FP32 = 0, EOT_BF16 = 1 } eot_dtype;

/* Kernel family.  AUTO picks the tensor-core (tcgen05/TMA) kernels for bf16 with d in
 * {64, 128} and a band that fits their shared-memory tile list (W up to about 7e4 when L is
 * longer than that; any W for shorter L), and the
 * CUDA-core kernels otherwise (fp32 is always computed on CUDA cores, in fp32, so that its
 * scores keep full fp32 precision).  TCGEN05 on a problem outside that range is
 * EOT_ERR_UNSUPPORTED. */
typedef enum { EOT_IMPL_AUTO = 0, EOT_IMPL_SIMT = 1, EOT_IMPL_TCGEN05 = 2 } eot_impl;

typedef struct {
    int32_t B, H;          /* batch, heads */
    int32_t L;             /* sequence length incl. dustbin and fillers; multiple of 128 */
    int32_t d;             /* head dim: multiple of 8, <= 128 (tensor-core path: 64 or 128) */
    int32_t W;             /* band width: support |i - j| <= W / 2 (integer division), W >= 0 */
    int32_t T;             /* stopped base steps, T >= 0 */
    int32_t R;             /* differentiable tail steps, 0 <= R <= 8 */
    int32_t dtype;         /* eot_dtype of Q, K, V, O, dO, dQ, dK, dV; potentials are fp32 */
    float scale;           /* score scale; 0 means 1 / sqrt(d) */
    int32_t dustbin;       /* 0 or 1 */
    int32_t dustbin_index; /* position of the dustbin token (0 <= index < L) when dustbin = 1 */
    float dustbin_mass;    /* dustbin marginal in [0, 1); 0 makes the dustbin inactive */
    int32_t dustbin_self;  /* 1: (D, D) is in the support; 0: it is not */
    int32_t impl;          /* eot_impl */
} eot_problem;

/* Bytes of device workspace that eot_sinkhorn_fwd (for_backward = 0) or eot_sinkhorn_bwd
 * (for_backward = 1) needs for problem *p.  Returns 0 when *p is invalid (see
 * eot_validate) and for empty problems.  Workspace must be 256-byte aligned. */
size_t eot_workspace_bytes(const eot_problem* p, int for_backward);

/* Host-side validation only: EOT_OK, EOT_ERR_INVALID_ARGUMENT or EOT_ERR_UNSUPPORTED. */
eot_status eot_validate(const eot_problem* p);

/*
 * Forward (§2.1).  Device pointers:
 *   Q, K, V   [B, H, L, d] dtype, read only.
 *   mask      [B, L] uint8, 1 = active real token; NULL = every position active.  With a
 *             dustbin, the dustbin position and everything after it are ignored in the mask
 *             (the dustbin is active iff mass > 0 and at least one real token is active;
 *             positions after it are inactive fillers).
 *   O         [B, H, L, d] dtype, written.  O_i = (1/a_i) sum_j P_ij V_j.
 *   u_tail    [B, H, R+1, L] float32, written: u_tail[0] = u after the T base steps (0 when
 *             T = 0), u_tail[k] = u(k) of tail step k.
 *   v_tail    [B, H, R+1, L] float32, written: v_tail[0] = stopped base v0, v_tail[k] = v(k).
 *   workspace eot_workspace_bytes(p, 0) bytes, device, contents clobbered.
 */
eot_status eot_sinkhorn_fwd(const eot_problem* p, const void* Q, const void* K, const void* V,
                            const uint8_t* mask, void* O, float* u_tail, float* v_tail,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward: exact adjoint of the R-step tail w.r.t. Q, K, V, the base (u0, v0) held fixed
 * (stop-gradient, §2.1-§2.2), for the loss gradient dO.  Inputs as in the forward plus
 * u_tail/v_tail from it and dO [B, H, L, d].  dQ, dK, dV [B, H, L, d] are overwritten (not
 * accumulated).  The gradient w.r.t. the dustbin token is written at ``dustbin_index`` per
 * (batch, head); a caller sharing one learned token across the batch sums over B.
 */
eot_status eot_sinkhorn_bwd(const eot_problem* p, const void* Q, const void* K, const void* V,
                            const uint8_t* mask, const float* u_tail, const float* v_tail,
                            const void* dO, void* dQ, void* dK, void* dV, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * One half-step of the band iteration (§2.1) on its own: the step each rank takes when one
 * unit's sequence is split over several devices (each part updates its own positions from the
 * potentials over its halo, and the parts exchange their boundary values between half-steps).
 * For every unit (b, h) and every position i with log_marg[b, i] > -inf:
 *     out[b, h, i] = log_marg[b, i]
 *                    - log sum_{j : |i - j| <= W / 2, log_marg[b, j] > -inf}
 *                          exp( scale * <X[b, h, i], Y[b, h, j]> + in[b, h, j] )
 * and out[b, h, i] = 0 where log_marg[b, i] = -inf.  A row half-step (u from v) passes X = Q,
 * Y = K, in = v; a column half-step (v from u) passes X = K, Y = Q, in = u.  The sum keeps a
 * running maximum, so any finite input potential is accepted.  Device pointers:
 *   X, Y      [B, H, L, d] p->dtype, read only.
 *   log_marg  [B, L] float32 log marginals, -inf for positions outside the problem (inactive
 *             tokens, padding).  A part of a longer sequence passes the whole problem's
 *             marginals over its positions (they depend on the whole sequence's active count).
 *   in        [B, H, L] float32, read only (ignored where log_marg is -inf).
 *   out       [B, H, L] float32, written.
 *   workspace eot_workspace_bytes(p, 0) bytes, 256-byte aligned, device, contents clobbered.
 * p->T and p->R are not used.  Errors, all returned before anything is launched except the
 * last: EOT_ERR_INVALID_ARGUMENT (invalid *p, a NULL pointer, a misaligned workspace),
 * EOT_ERR_UNSUPPORTED (p->dustbin = 1: the dustbin's dense row and column sum over every
 * position, which a part cannot form alone), EOT_ERR_WORKSPACE_TOO_SMALL, EOT_ERR_CUDA.
 * Asynchronous on ``stream``; the device status word is read with eot_last_device_status.
 */
eot_status eot_band_half_step(const eot_problem* p, const void* X, const void* Y, const float* log_marg,
                              const float* in, float* out, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * The same half-step for a part of a sequence that carries a dustbin (§2.3; p->dustbin = 1,
 * D = p->dustbin_index, positions after D inactive).  The dustbin is linked to every active real
 * position of the whole sequence, so its row and column are dense over all parts:
 *   - every active real position i < D gets out[b, h, i] as in eot_band_half_step with the
 *     dustbin term exp(scale * <X_i, Y_D> + in_D) added to its sum;
 *   - instead of a finished out[b, h, D], the part's share of the dustbin's sum over the
 *     positions it owns, [own_lo, own_hi) (0 <= own_lo <= own_hi <= D), excluding (D, D):
 *       x_c = scale * <X[b, h, D], Y[b, h, c]> + in[b, h, c]  over active c in [own_lo, own_hi),
 *       dust_part[b, h, 0] = M = max_c x_c,  dust_part[b, h, 1] = sum_c exp(x_c - M)
 *     ((-inf, 0) when the range holds no active position).  The caller merges the parts'
 *     partials (a max and a sum over all parts), adds the (D, D) term when it is in the support,
 *     and forms out_D = log_marg[D] - (M + log(sum)); out[b, h, D] is left unspecified.
 *   log_marg[b, D] is the dustbin's log marginal (log mass), the real positions' the whole
 *   problem's (log((1 - mass) / n_real)).  dust_part: [B, H, 2] float32, device, written.
 * Other arguments, errors and asynchrony as for eot_band_half_step; p->dustbin = 0 or an own range
 * outside [0, D] is EOT_ERR_INVALID_ARGUMENT.
 */
eot_status eot_band_half_step_dustbin(const eot_problem* p, const void* X, const void* Y,
                                      const float* log_marg, const float* in, float* out, int32_t own_lo,
                                      int32_t own_hi, float* dust_part, void* workspace,
                                      size_t workspace_bytes, void* stream);

/*
 * The output of given potentials (§2.1) on its own, the last step of a sequence-sharded forward
 * (each part forms the rows it owns from the potentials over its halo):
 *     O[b, h, i] = (1 / a_i) sum_{j : |i - j| <= W / 2, active j}
 *                      exp( scale * <Q[b, h, i], K[b, h, j]> + u[b, h, i] + v[b, h, j] ) V[b, h, j]
 * with a_i = exp(log_marg[b, i]) for active i; O = 0 at inactive positions.  Device pointers:
 *   Q, K, V   [B, H, L, d] p->dtype, read only;
 *   log_marg  [B, L] float32 log marginals (-inf = inactive; a part passes the whole problem's);
 *   u, v      [B, H, L] float32 potentials, read only;
 *   O         [B, H, L, d] p->dtype, written;
 *   workspace eot_workspace_bytes(p, 0) bytes, 256-byte aligned, device, contents clobbered.
 * p->T and p->R are not used; a dustbin is EOT_ERR_UNSUPPORTED (its dense output row sums over
 * every position).  Errors and asynchrony as for eot_band_half_step.
 */
eot_status eot_band_output(const eot_problem* p, const void* Q, const void* K, const void* V,
                           const float* log_marg, const float* u, const float* v, void* O, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Synchronises ``stream``, reads the device status word that the last fwd/bwd call on this
 * workspace left, clears it, and returns EOT_OK, EOT_ERR_NONFINITE or EOT_ERR_TIMEOUT
 * (EOT_ERR_CUDA if the copy fails). */
eot_status eot_last_device_status(void* workspace, void* stream);

/* Raw device status bits of the last call (bit 0 non-finite, bit 1 timeout); syncs. */
eot_status eot_device_status_bits(void* workspace, void* stream, uint32_t* bits);

/* Static string for a status code. */
const char* eot_status_string(eot_status s);

/* EOT_ABI_VERSION of the loaded library. */
int eot_abi_version(void);

/* Benchmark support (process-wide, not thread-safe).
 * eot_kernel_launches: number of kernels this library has enqueued since it was loaded.
 * eot_profile_begin / eot_profile_end: between the two calls, every sweep that fwd/bwd
 * enqueue is bracketed by a pair of CUDA events recorded on the call's stream;
 * eot_profile_end synchronises ``stream`` and totals the elapsed times per kind.
 * eot_profile_read(kind, ...): kind 0 = forward half-step sweeps, 1 = forward output sweep,
 * 2 = backward sweeps other than the staircase, 3 = auxiliary kernels (marginals, vectors,
 * dustbin links), 4 = the staircase sweeps of the backward (R >= 2); returns
 * the summed milliseconds and the number of bracketed launches of that kind. */
long long eot_kernel_launches(void);
/* Exponentials per band entry that the forward solve (base and tail, not the output sweep)
 * evaluates for problem *p under the current forward schedule: 2 (T + R) when every half-step
 * forms its own plan entries, T + R + 1 when each iteration forms them once; -1 for an invalid
 * problem.  Benchmark support: the exponential-unit bound of the solve. */
int eot_solve_exp_passes(const eot_problem* p);
/* Forward schedule for every later call in this process (benchmark and test support):
 *   0, 1  the half-step schedule: every half-step forms the plan entries of its band once (two
 *         exponentials per band entry per iteration).  0 is the default; it is the faster schedule
 *         on every workload measured (a B200 at 1965 MHz: the long workload's solve 5.05 ms against
 *         8.25 ms, the medium 1.12 against 1.85 ms, the protein-like 2.45 against 3.97 ms);
 *   2     one exponential per band entry per iteration (row sums in registers, column sums on the
 *         tensor core from the entries kept on chip) for bf16 problems without a dustbin, T >= 1,
 *         d in {64, 128} and a band whose 128-row strips meet at most nine 128-column tiles (W up
 *         to 1024), in one cooperative launch; a forward it cannot run returns EOT_ERR_UNSUPPORTED
 *         (EOT_ERR_CUDA if the device refuses the launch);
 *   3     the same with one launch per iteration (what 2 falls back to when the device refuses
 *         the cooperative launch).
 * Both schedules compute the same iterates; results differ by floating-point rounding only.
 * Returns EOT_ERR_INVALID_ARGUMENT for any other value. */
eot_status eot_set_forward_schedule(int schedule);
/* Backward schedule for every later workspace query and backward call in this process
 * (measurement support):
 *   0  every sweep recomputes the reference plan P(R,R) from S on the tensor cores (default; the
 *      extra memory stays O(L));
 *   1  the alpha_R row sweep also stores its plan entries as bf16 in a band store of
 *      B H L (2 (W/2) + 128) entries inside the workspace, and the staircase sweeps (R >= 2) stream
 *      it on CUDA cores instead of recomputing it: for tensor-core problems without a dustbin
 *      whose half-width W/2 is a multiple of 128; others run schedule 0.
 * eot_workspace_bytes(p, 1) includes the band store only under schedule 1.  Returns
 * EOT_ERR_INVALID_ARGUMENT for any other value. */
eot_status eot_set_backward_schedule(int schedule);
void eot_profile_begin(void);
eot_status eot_profile_end(void* stream);
eot_status eot_profile_read(int kind, double* total_ms, long long* launches);

/* Forward pass that allocates nothing and takes no workspace.  The paper has no counterpart:
 * this is a deployment variant of eot_sinkhorn_fwd for callers that cannot allocate device
 * memory where they run it (a plug-in inside a host that owns all device memory and gives it
 * no allocator; a serving loop that forbids cudaMalloc/cudaFree after start-up because those
 * calls can synchronise the device).  Arguments and results are those of eot_sinkhorn_fwd;
 * the scratch is a fixed array of EOT_STATIC_SCRATCH_BYTES in this library's device memory.
 *   - The array belongs to each context that loads this library's kernels and is held until
 *     the module is unloaded (normally process exit).  Every call looks up its address in the
 *     context current at that moment (cudaGetSymbolAddress, a host-side query that allocates
 *     nothing), so callers that switch contexts or reset the device stay correct.
 *   - The first call in a context loads the library's kernels there (CUDA lazy module loading),
 *     which may allocate device memory for the module and is not allowed during stream capture:
 *     make one call before any capture and before the phase in which nothing may allocate.
 *     Later calls allocate nothing.
 *   - Problems whose forward scratch, eot_workspace_bytes(p, 0), exceeds
 *     EOT_STATIC_SCRATCH_BYTES are rejected with EOT_ERR_WORKSPACE_TOO_SMALL before anything
 *     is launched.
 *   - Every call in a context shares the one array and leaves its contents behind (the first
 *     kernel of each call clears what must start at zero).  Calls that overlap on the GPU
 *     (other streams, other host threads) race on it and corrupt each other: serialise them.
 *   - The device status word of these calls lives in the shared array: read (and clear) it
 *     with eot_static_last_device_status, which syncs ``stream`` like eot_last_device_status.
 * eot_static_scratch_bytes returns EOT_STATIC_SCRATCH_BYTES as built into the library. */
#define EOT_STATIC_SCRATCH_BYTES (32u * 1024u * 1024u)
eot_status eot_sinkhorn_fwd_static(const eot_problem* p, const void* Q, const void* K, const void* V,
                                   const uint8_t* mask, void* O, float* u_tail, float* v_tail,
                                   void* stream);
eot_status eot_static_last_device_status(void* stream);
size_t eot_static_scratch_bytes(void);

/* Self-test of the bounded device waits (failure detection; the paper has no counterpart).
 * Every wait inside this library's kernels (on an mbarrier, or on a grid-wide counter between
 * fused half-steps) gives up after a time limit, sets the timeout bit of the status word and
 * ends the kernel instead of spinning forever.  This call runs one tiny kernel whose single
 * wait, with limit ``limit_ns`` (1 ns .. 1 s), is made so that nothing completes it:
 *   EOT_SELFTEST_MBARRIER  an mbarrier expecting two arrivals receives one;
 *   EOT_SELFTEST_GRID      a grid-wide counter waits for one CTA more than the grid holds;
 *   EOT_SELFTEST_CONTROL   the mbarrier receives both arrivals (the wait completes at once).
 * ``scratch`` is a caller-owned device buffer of at least 256 bytes, 256-byte aligned: word 0
 * is the status word (read it with eot_last_device_status(scratch, stream): EOT_ERR_TIMEOUT for
 * the first two cases, EOT_OK for the control), word 2 is 2 when the wait gave up and 1 when it
 * completed.  Asynchronous on ``stream``; invalid arguments return EOT_ERR_INVALID_ARGUMENT
 * before anything is enqueued. */
#define EOT_SELFTEST_MBARRIER 0
#define EOT_SELFTEST_GRID 1
#define EOT_SELFTEST_CONTROL 2
eot_status eot_wait_selftest(int which, uint64_t limit_ns, void* scratch, void* stream);

/* Kernel family that ``p`` would run with (EOT_IMPL_SIMT or EOT_IMPL_TCGEN05), or -1 if
 * the problem is invalid or unsupported. */
int eot_resolved_impl(const eot_problem* p);

/* Norms for the a-posteriori bias certificate of the tail ("Blockwise Differentiable Sinkhorn
 * Attention" §2.4, third certificate: measure how far the tail gradient is from the gradient
 * through the whole solve, and choose the tail depth from it).  Accumulates, in float64,
 *     out[0] = sum_i (a_i - b_i)^2,    out[1] = sum_i a_i^2
 * over the n elements of the device arrays a and b (element type ``dtype``, e.g. two tail
 * gradients).  ``out`` is a device array of two doubles, overwritten.  Stream-ordered and
 * asynchronous; the summation order varies between runs (float64 atomics), so the last bits
 * may too.  Null pointers (a, b with n > 0) or an unknown dtype return
 * EOT_ERR_INVALID_ARGUMENT before anything is enqueued; a launch failure EOT_ERR_CUDA. */
eot_status eot_sq_norms(const void* a, const void* b, size_t n, eot_dtype dtype, double* out, void* stream);

/* Projective contraction certificate ("Blockwise Differentiable Sinkhorn Attention" §2.4, second
 * certificate: with Hilbert's projective metric, the strictly positive active blocks of the
 * Sinkhorn map are contractions).  For every pair of 128-position tiles I (positions
 * [128 I, 128 I + 128)) and J = I + o that lies wholly inside the band, |o| * 128 + 127 <= W / 2,
 * the Birkhoff-Hopf ratio of the block exp(S) on its active real tokens:
 *     kappa = tanh(Delta / 4),  Delta = max over rows i, i' and columns j, j' of
 *                                       S_ij + S_i'j' - S_ij' - S_i'j,
 * S = scale Q K^T formed in float32.  kappa is a caller-owned device float32 array
 * [B, H, ceil(L / 128), n] with n = eot_contraction_offsets(p) = 2 m + 1 entries per tile
 * (offset o at index o + m), -1 where J is out of range or the block has no active row or
 * column.  Q, K and mask are those of eot_sinkhorn_fwd (p->dtype; the dustbin and the fillers
 * after it are left out of every block); T and R are not used.  No workspace; stream-ordered and
 * asynchronous.  eot_contraction_offsets returns 0 when no tile pair fits in the band (then
 * eot_contraction writes nothing) and -1 for an invalid problem; eot_contraction reports
 * argument errors as eot_sinkhorn_fwd does, before anything is enqueued. */
int eot_contraction_offsets(const eot_problem* p);
eot_status eot_contraction(const eot_problem* p, const void* Q, const void* K, const uint8_t* mask, float* kappa,
                           void* stream);

#ifdef __cplusplus
}
#endif

#endif /* EOT_H_ */
