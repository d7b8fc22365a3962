/*
 * sinkhorn_attn.h -- C ABI of the B200 (sm_100a) banded log-domain Sinkhorn
 * attention library (libsinkhorn_attn.so).
 *
 * The operation (Block-Wise Differentiable Sinkhorn Attention; gist.science/de
 * and gist.science/fr technical summaries, sections 2.1-2.3; abstracts on
 * dzcademia.com and searcharxiv.com):
 *
 *   S_ij = <q_i, k_j> / (sqrt(d) * eps) on the band
 *   Omega = {(i, j) : |i - j| <= W, mask_i = mask_j = 1}.
 *   Stopped base: v = 0, then T iterations of
 *       u_i <- -log sum_{j in Omega_i} exp(S_ij + v_j)      (rows first)
 *       v_j <- -log sum_{i in Omega_j} exp(S_ij + u_i)      (then columns)
 *   giving (u0, v0), held constant under differentiation.
 *   Tail: R more iterations of the same update from v0, giving u1, v1, ..., uR, vR.
 *   O = P^(R,R) V with P^(a,b)_ij = exp(S_ij + u^(a)_i + v^(b)_j) on Omega.
 *   Backward: the exact vector-Jacobian product of the tail with respect to
 *   Q, K, V for an arbitrary cotangent dO (section 2.2; R = 2 has the four
 *   staircase plans P^(2,2), P^(2,1), P^(1,1), P^(1,0)).
 *   Dustbin (section 2.3): the same surrogate on a support enlarged by one
 *   dustbin row and one dustbin column (plus their corner) carrying the
 *   constant score dustbin_score, with unit mass like every other row/column.
 *
 * Debug build: compiled with -DSA_DEBUG (libsinkhorn_attn_debug.so) every
 * kernel checks the indices of its guarded accesses (global rows and columns,
 * ring and buffer slots, tensor-memory columns, shared-memory offsets) before
 * making them; a failed check skips the access and records SA_ERR_BOUNDS in
 * the status word (read by sinkhorn_attn_poll).  Nothing traps.
 *
 * Conventions shared by every entry point
 *   - The caller owns every buffer.  The library allocates no device or host
 *     memory in any call and keeps no mutable global state, so concurrent
 *     calls on different buffers are safe (sinkhorn_attn_bwd_static_ws is the
 *     one exception: it uses a fixed scratch array inside the library).
 *   - Device pointers must be 16-byte aligned, point to device memory of the
 *     current device (or to managed memory), and the tensors be contiguous in
 *     the stated layout; otherwise the call returns SA_ERR_INVALID_ARG before
 *     launching anything.  Page-locked host memory and another GPU's memory
 *     are rejected (make the tensors' device current before the call).
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL means
 *     the legacy default stream).  Argument and launch errors are returned at
 *     once.  The tensor-core sweeps and the O(L) kernels between them are
 *     launched with programmatic stream serialisation (a kernel's set-up may
 *     overlap the end of the kernel before it on the stream, and it waits for
 *     that kernel to complete before it touches global memory); the other
 *     kernels are ordinary launches.  Either way the ordering against the
 *     caller's own work on the stream is that of ordinary launches.
 *     Conditions found on the device (a non-finite dual or output when
 *     check_finite is set) are recorded in a status word at the start of the
 *     workspace and returned by sinkhorn_attn_poll().
 *   - Masked tokens (mask_i == 0) have exactly zero duals, O, dQ, dK and dV.
 *   - Tensors Q, K, V, O, dO, dQ, dK, dV are [B][H][L][d] row-major with d
 *     contiguous, of element type `dtype`.  Duals are float32.
 */
#ifndef SINKHORN_ATTN_H
#define SINKHORN_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SA_OK = 0,
    SA_ERR_INVALID_ARG = -1,  /* null/misaligned pointer, bad size or parameter */
    SA_ERR_UNSUPPORTED = -2,  /* valid request outside what this build implements */
    SA_ERR_WORKSPACE = -3,    /* workspace smaller than sinkhorn_attn_workspace_size() */
    SA_ERR_CUDA = -4,         /* a CUDA runtime call or kernel launch failed */
    SA_ERR_NONFINITE = -5,    /* device found a NaN/Inf (only with check_finite) */
    SA_ERR_TIMEOUT = -6,      /* a bounded device-side wait gave up */
    SA_ERR_EXCHANGE = -7,     /* a sharded call's halo exchange callback failed */
    SA_ERR_BOUNDS = -8        /* debug build only: a device-side bounds check failed */
} sa_status;

typedef enum { SA_F32 = 0, SA_BF16 = 1 } sa_dtype;

/* Backward schedule (section 2.2).  ONE_REFERENCE forms only P^(R,R) and
 * rescales it with exp(u^(a)-u^(R)) exp(v^(b)-v^(R)); DIRECT forms every
 * staircase plan with its own exponential (the direct-four adjoint for R=2). */
typedef enum { SA_BWD_ONE_REFERENCE = 0, SA_BWD_DIRECT = 1 } sa_bwd_schedule;

typedef struct {
    int B, H, L, d;        /* batch, heads, sequence length, head dim (d == 64) */
    int W;                 /* band half-width, W >= 0 (W >= L-1 is dense) */
    float eps;             /* entropic temperature, > 0 */
    int T;                 /* stopped base iterations, T >= 0 */
    int R;                 /* differentiable tail iterations, 0 <= R <= 256 (2 in the
                              pages); the forward needs T + R >= 1 (the backward does
                              not read T).  T = 0, R = N backpropagates through
                              the whole N-iteration solve; R = 0 holds every dual
                              constant (dS = P * dO V^T, dV = P^T dO) */
    sa_dtype dtype;        /* element type of Q, K, V, O, dO, dQ, dK, dV */
    int dustbin;           /* 0 or 1: add the dustbin row and column */
    float dustbin_score;   /* score on every dustbin entry, used as given */
    sa_bwd_schedule bwd;   /* backward schedule */
    int check_finite;      /* 0 or 1: scan duals/outputs, set SA_ERR_NONFINITE */
    /* Optional launch trace for profiling (all NULL/0 to disable).  When
     * trace_cap > 0 the call records trace_events[2i] before and
     * trace_events[2i+1] after its i-th kernel launch on `stream` (cudaEvent_t
     * handles created by the caller), stores that launch's sa_kernel_kind in
     * trace_kinds[i] (host memory) for i < trace_cap, and writes the number
     * of launches it made to *trace_count (host memory, may be NULL). */
    void* const* trace_events;
    int* trace_kinds;
    int* trace_count;
    int trace_cap;
} sa_params;

/* Kernel kinds reported by the launch trace. */
typedef enum {
    SA_KERNEL_LSE_SWEEP = 1,   /* dual update: u <- -LSE_j(S+v) or v <- -LSE_i(S+u) */
    SA_KERNEL_PV = 2,          /* O = P V, or dV = P^T dO with vbar = rowdot(V, dV) */
    SA_KERNEL_WSUM = 3,        /* vector cotangent sweep: weighted plan row sums */
    SA_KERNEL_DS = 4,          /* dQ = c dS K or dK = c dS^T Q */
    SA_KERNEL_AUX = 5          /* O(L) elementwise helpers */
} sa_kernel_kind;

/* Number of float32 elements of the dual state: B*H*(2R+2)*(L+dustbin).
 * Layout [B][H][2R+2][L+dustbin]: row 2r is u^(r), row 2r+1 is v^(r),
 * r = 0..R; with a dustbin, index L of each row is the dustbin's dual.
 * Returns SA_ERR_INVALID_ARG for invalid params. */
sa_status sinkhorn_attn_state_size(const sa_params* p, size_t* n_floats);

/* Workspace bytes needed by sinkhorn_attn_fwd and sinkhorn_attn_bwd (either
 * pointer may be NULL).  Both are O(B*H*L) and include a 256-byte status
 * header at offset 0.  With bf16 storage and no dustbin (the tensor-core
 * path) both hold a working copy of the dual state: per dual, log2(e) times
 * its value as float32 and a bf16 [16] operand row per token (the dual divided
 * by the score scale, split in three bf16 parts), 36 bytes per token and dual.
 * The backward's grows with R (a few float32 vectors of B*H*(L+dustbin) per
 * tail step); it holds four bf16 [B][H][L][16] arrays (the modifier's
 * operands of the bf16 dS contraction, 128 bytes per token), and for R > 4 a
 * float32 [B][H][L][d] sum of the dQ / dK sweeps over blocks of at most 8
 * modifier terms. */
sa_status sinkhorn_attn_workspace_size(const sa_params* p, size_t* fwd_bytes, size_t* bwd_bytes);

/*
 * Forward (sections 2.1 and 2.3).
 *   q, k, v : [B][H][L][d] dtype, device.
 *   mask    : [B][L] uint8 (1 = valid, 0 = padding), device, or NULL (all valid).
 *   v_dust  : [H][d] float32 dustbin value vectors, device, or NULL (zero);
 *             read only when p->dustbin.
 *   o       : [B][H][L][d] dtype, device, written (masked rows = 0).
 *   state   : sinkhorn_attn_state_size() float32, device, written.
 *   ws      : workspace of ws_bytes >= fwd_bytes, device.
 * Score tiles are recomputed in every sweep; nothing of size L*W is stored.
 */
sa_status sinkhorn_attn_fwd(const sa_params* p, const void* q, const void* k, const void* v,
                            const uint8_t* mask, const float* v_dust, void* o, float* state,
                            void* ws, size_t ws_bytes, void* stream);

/*
 * Backward: dQ, dK, dV (and the dustbin's value and score gradients) of
 * <dO, O> through the R-step tail, the stopped base held constant (section 2.2;
 * the dustbin token of section 2.3 is learned: its value vector and its score).
 *   q, k, v, mask, v_dust : as given to the forward.
 *   o, state              : the forward's outputs.
 *   dO                    : [B][H][L][d] dtype, device.
 *   dq, dk, dv            : [B][H][L][d] dtype, device, written.
 *   dv_dust               : [H][d] float32, device, written (summed over the
 *                           batch), or NULL; used only when p->dustbin.
 *   d_dust_score          : one float32, device (4-byte aligned), written with
 *                           the cotangent of p->dustbin_score summed over every
 *                           (batch, head) problem, or NULL; used only when
 *                           p->dustbin.  The score enters every dustbin entry
 *                           (column, row, corner), so this is the sum of the
 *                           score cotangent over them, each staircase plan on
 *                           those O(L) entries formed by its own exponential
 *                           whatever the schedule.
 *   ws                    : workspace of ws_bytes >= bwd_bytes, device.
 * The schedule is p->bwd.
 */
sa_status sinkhorn_attn_bwd(const sa_params* p, const void* q, const void* k, const void* v,
                            const uint8_t* mask, const float* v_dust, const void* o,
                            const void* dO, const float* state, void* dq, void* dk, void* dv,
                            float* dv_dust, float* d_dust_score, void* ws, size_t ws_bytes,
                            void* stream);

/*
 * Sequence sharding (no counterpart in the pages, which shard by batch): one
 * problem's tokens split into contiguous shards, one per rank, each rank
 * holding its own tokens plus halos of its neighbours' tokens.  The local
 * sequence of p->L tokens is
 *     [0, halo_lo)                 the left neighbour's last halo_lo tokens,
 *     [halo_lo, L - halo_hi)       this rank's own tokens,
 *     [L - halo_hi, L)             the right neighbour's first halo_hi tokens,
 * with halo_lo = 0 on the shard that starts the sequence and halo_hi = 0 on
 * the one that ends it; an interior halo must hold at least W tokens (every
 * band neighbour of an own token is then local) and every shard at least W
 * own tokens (a halo then comes from one neighbour).  The sharded calls run the
 * same sweeps as the unsharded ones, and after every sweep that produces a dual
 * or vector cotangent they call
 *     exchange(vec, row_stride, rows, user, stream)
 * on the host, in stream order (the sweep has been launched on `stream`, not
 * necessarily finished): vec + r * row_stride (r < rows = B*H) is row r's p->L
 * float32 entries in device memory, and the callback must, before returning
 * or in work it enqueues on `stream`, overwrite each row's halo entries with
 * the values its neighbours hold for those tokens (and hand them this rank's
 * edge values).  Every rank makes the same sequence of calls.  A non-zero
 * return ends the call with SA_ERR_EXCHANGE.  Results are exact for own
 * tokens; halo rows of o, dq, dk, dv hold partial values to be discarded.
 * The dustbin couples every token and is not supported (SA_ERR_UNSUPPORTED).
 */
typedef int (*sa_exchange_fn)(float* vec, long long row_stride, int rows, void* user,
                              void* stream);
typedef struct {
    int halo_lo, halo_hi;      /* halo tokens at the start and end of the local sequence */
    sa_exchange_fn exchange;   /* not NULL */
    void* user;                /* passed through to exchange */
} sa_shard;

/* sinkhorn_attn_fwd / sinkhorn_attn_bwd on one shard of a sequence-sharded
 * problem (see sa_shard); the other arguments, sizes and the workspace are
 * those of the unsharded calls for the local sequence length p->L.
 * SA_ERR_INVALID_ARG for a NULL shard or exchange, or halos outside [0, L]
 * that overlap; SA_ERR_UNSUPPORTED with a dustbin. */
sa_status sinkhorn_attn_fwd_sharded(const sa_params* p, const sa_shard* shard, const void* q,
                                    const void* k, const void* v, const uint8_t* mask, void* o,
                                    float* state, void* ws, size_t ws_bytes, void* stream);
sa_status sinkhorn_attn_bwd_sharded(const sa_params* p, const sa_shard* shard, const void* q,
                                    const void* k, const void* v, const uint8_t* mask,
                                    const void* o, const void* dO, const float* state, void* dq,
                                    void* dk, void* dv, void* ws, size_t ws_bytes, void* stream);

/*
 * One forward + backward step with inputs and results in host memory (no
 * counterpart in the pages).  Every (batch, head) problem is independent, so
 * the problems are split into `groups` contiguous groups (whole batches, or
 * runs of heads within one batch when there are fewer batches than groups;
 * whole batches with a dustbin) and pipelined: group g+1's inputs are copied
 * to the device and group g-1's results back while group g runs
 * sinkhorn_attn_fwd and sinkhorn_attn_bwd, on two copy streams of the library
 * ordered against `stream` with events.  Host buffers should be page-locked
 * (cudaHostAlloc / cudaHostRegister) for the copies to overlap; pageable
 * memory works, serialised by the driver.  The call returns once everything is
 * enqueued; the results are in host memory when `stream` reaches that point
 * (synchronise it before reading them).  The two copy streams are created
 * (non-blocking) on a device's first call and kept for the life of the
 * process; calls on one device share them, so overlapping calls serialise
 * their copies.
 */
typedef struct {
    const void *q, *k, *v, *dO;  /* host [B][H][L][d] dtype */
    const uint8_t* mask;         /* host [B][L] uint8, or NULL (all valid) */
    const float* v_dust;         /* host [H][d] float32, or NULL (zero); dustbin only */
    void *o, *dq, *dk, *dv;      /* host [B][H][L][d] dtype, written */
    float* state;                /* host [B][H][2R+2][L+dustbin] float32, written, or NULL */
    float* dv_dust;              /* host [H][d] float32, written, or NULL; dustbin only */
    float* d_dust_score;         /* host, one float32, written, or NULL; dustbin only */
    int groups;                  /* >= 1; 3-8 overlap copies with compute */
} sa_host_step;

/* Device workspace bytes for sinkhorn_attn_step_host with `groups` groups:
 * two groups' device copies of inputs and results plus their fwd/bwd
 * workspaces. */
sa_status sinkhorn_attn_step_host_workspace_size(const sa_params* p, int groups, size_t* bytes);

/* SA_ERR_INVALID_ARG for a device pointer where host memory is expected, a NULL
 * input or output, or groups < 1; SA_ERR_UNSUPPORTED with check_finite;
 * SA_ERR_WORKSPACE below the size above; otherwise the statuses of the
 * forward and backward. */
sa_status sinkhorn_attn_step_host(const sa_params* p, const sa_host_step* io, void* ws,
                                  size_t ws_bytes, void* stream);

/*
 * Test hook: the plan P^(a,b) (0 <= a, b <= R) from a finished forward state.
 *   band : [B][H][L][2W+1] float32, entry t of row i is column i-W+t (0 off Omega).
 *   dcol : [B][H][L] float32 entries (i, dustbin), or NULL.
 *   drow : [B][H][L+1] float32 entries (dustbin, j), corner last, or NULL.
 * dcol/drow are written only when p->dustbin.
 */
sa_status sinkhorn_attn_debug_plan(const sa_params* p, int a, int b, const void* q,
                                   const void* k, const uint8_t* mask, const float* state,
                                   float* band, float* dcol, float* drow, void* stream);

/*
 * Backward without caller-provided workspace.  No counterpart in the paper:
 * this exists for callers that cannot allocate device memory at the point
 * where they run the backward -- for example a host framework that owns all
 * device memory and forbids allocations inside its step, or latency-critical
 * code that cannot afford cudaMalloc's implicit device-wide synchronisation --
 * and that have no spare buffer to lend as workspace.
 *
 * Same arguments, layouts and results as sinkhorn_attn_bwd, minus ws and
 * ws_bytes.  The scratch comes from one fixed array of
 * SA_STATIC_SCRATCH_BYTES bytes compiled into the library; every GPU that
 * loads the library holds it until the process exits.  Problems whose
 * backward workspace (sinkhorn_attn_workspace_size) exceeds that size are
 * rejected with SA_ERR_WORKSPACE before anything is launched.
 *   - The call allocates nothing: no cudaMalloc/cudaFree or allocating
 *     library routine.
 *   - Every call looks up the array's device address on the current device
 *     (make the tensors' device current); the lookup allocates nothing.  The
 *     first call on a device may load the library's module on it, so make
 *     that first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents, so
 *     calls whose work overlaps on the GPU (different streams, or different
 *     host threads on one device) race: serialise them.
 *   - Conditions found on the device (a bounded wait that gave up:
 *     SA_ERR_TIMEOUT) go to the status word at the start of the array, where
 *     they stay, across calls, until sinkhorn_attn_poll_static() reads and
 *     resets them; poll after the calls whose results you use.
 *   - check_finite is not supported here: SA_ERR_UNSUPPORTED.
 */
#define SA_STATIC_SCRATCH_BYTES (32u << 20)
sa_status sinkhorn_attn_bwd_static_ws(const sa_params* p, const void* q, const void* k,
                                      const void* v, const uint8_t* mask, const float* v_dust,
                                      const void* o, const void* dO, const float* state,
                                      void* dq, void* dk, void* dv, float* dv_dust,
                                      float* d_dust_score, void* stream);

/* Synchronises `stream`, then returns the status word recorded in `ws` by the
 * last forward/backward that used it (SA_OK, SA_ERR_NONFINITE or
 * SA_ERR_TIMEOUT) and resets it to SA_OK. */
sa_status sinkhorn_attn_poll(void* ws, void* stream);

/* sinkhorn_attn_poll for the fixed scratch array of
 * sinkhorn_attn_bwd_static_ws on the current device: synchronises `stream`,
 * returns the status word that the static-scratch backward calls have recorded
 * since the last poll (SA_OK or SA_ERR_TIMEOUT), and resets it to SA_OK.
 * No counterpart in the paper (see sinkhorn_attn_bwd_static_ws).  Returns
 * SA_ERR_CUDA if the array's address cannot be looked up. */
sa_status sinkhorn_attn_poll_static(void* stream);

/* Static English description of a status code. */
const char* sinkhorn_attn_strerror(sa_status s);

/* Squared distance for the a-posteriori bias certificate (gist.science/de
 * section 3, section 4.1): the certificate of tail depth R compares the
 * gradients with T = N - R stopped iterations against full backpropagation
 * (T = 0, R = N) as ||g_R - g_full|| / ||g_full||.  This call supplies the two
 * sums for one gradient tensor:
 *   out[0] = sum_i (x_i - y_i)^2,  out[1] = sum_i y_i^2,
 * accumulated in double over n elements of type dtype (SA_F32 or SA_BF16).
 *   x, y : n elements each, device, 16-byte aligned (may be NULL when n == 0).
 *   out  : 2 doubles, device, 16-byte aligned; zeroed on `stream`, then
 *          written by the kernel (summation order is not fixed, so the last
 *          bits may differ between calls).
 * Returns SA_ERR_INVALID_ARG for n < 0, another dtype, or a bad pointer;
 * SA_ERR_CUDA on a launch error; else SA_OK. */
sa_status sinkhorn_attn_sq_dist(const void* x, const void* y, long long n, sa_dtype dtype,
                               double* out, void* stream);

/* The a-posteriori bias certificate from the squared distances (gist.science/de
 * section 3, section 4.1): for tail depth R the certificate is
 *     eta_R = ||g_R - g_full|| / ||g_full||
 * over all gradient tensors together (dQ, dK, dV), g_R the gradients with
 * T = N - R stopped iterations and g_full full backpropagation (T = 0, R = N);
 * the depth the pages select at tolerance tau is the smallest R with
 * eta_R <= tau.  Host-only arithmetic (no device work).
 *   depths : n_depths tail depths R (>= 0), host.
 *   sums   : [n_depths][n_tensors][2] doubles, host: entry (i, t) holds
 *            sinkhorn_attn_sq_dist's (sum (x - y)^2, sum y^2) for tensor t with
 *            x from depth depths[i] and y from full backpropagation.
 *   eta    : n_depths doubles, host, written (eta = ||x - y|| when every
 *            ||y|| is 0).
 *   r_star : one int, host, written: the smallest depth with eta <= tau, or -1.
 * Returns SA_ERR_INVALID_ARG for n_depths or n_tensors < 1, a NULL pointer, a
 * negative depth, tau < 0 or NaN, or a negative or NaN sum; else SA_OK. */
sa_status sinkhorn_attn_bias_certificate(int n_depths, const int* depths, int n_tensors,
                                         const double* sums, double tau, double* eta,
                                         int* r_star);

/* Test hook for the exponentials of the row-sum sweeps (the dual updates and
 * the vector-cotangent sweeps); no counterpart in the pages.  For each of the
 * n float32 arguments x (x <= 0; device, 4-byte aligned) it writes 2^x as those
 * sweeps evaluate it on the FMA pipe (y_poly: round-to-nearest range
 * reduction and a degree-5 polynomial, arguments clamped at -126) and on the
 * MUFU unit (y_mufu: ex2.approx).  Returns SA_ERR_INVALID_ARG for n < 0 or a
 * pointer that is not device memory of the current device, SA_ERR_CUDA on a
 * launch error, else SA_OK. */
sa_status sinkhorn_attn_debug_exp2(const float* x, long long n, float* y_poly, float* y_mufu,
                                   void* stream);

/* Test hook for the failure path; no counterpart in the pages.  Launches on
 * `stream` one CTA whose thread waits, through the same bounded mbarrier wait
 * every kernel of this library uses, on a barrier that nothing ever arrives on;
 * after `budget_cycles` SM clock cycles (clamped to [1, 1e8], at most about
 * 50 ms) the wait gives up and records SA_ERR_TIMEOUT in the status word of
 * `ws` (a workspace of at least 256 bytes, device memory), exactly as a
 * stalled pipeline stage would.  Nothing faults and the CUDA context stays
 * usable; sinkhorn_attn_poll(ws, stream) then returns SA_ERR_TIMEOUT.
 * With ws == NULL the timeout is recorded in the status word of the fixed
 * scratch array of sinkhorn_attn_bwd_static_ws on the current device, and
 * sinkhorn_attn_poll_static(stream) returns it.
 * Returns SA_ERR_INVALID_ARG for a misaligned `ws` or one that is not device
 * memory of the current device, SA_ERR_CUDA on a launch error, else SA_OK. */
sa_status sinkhorn_attn_debug_timeout(void* ws, long long budget_cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SINKHORN_ATTN_H */
