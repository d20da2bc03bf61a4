/*
 * ssm_scan.h -- C ABI of the B200 (sm_100a) selective-scan library (libssm_scan.so).
 *
 * The operation (Mamba selective scan).  For every sequence b, channel d and state n:
 *
 *     Delta_t = softplus(delta[b,d,t] + delta_bias[d])
 *     h_t[n]  = exp(Delta_t * A[d,n]) * h_{t-1}[n] + Delta_t * B[b,n,t] * u[b,d,t]
 *     y[b,d,t] = (sum_n C[b,n,t] * h_t[n] + Dskip[d] * u[b,d,t]) * silu(z[b,d,t])
 *
 * (with `discretization = SSM_DISC_ZOH` the input term Delta_t * B is replaced by the
 * zero-order hold's (exp(Delta_t A[d,n]) - 1) / A[d,n] * B; see ssm_discretization_t)
 *
 * Sources (web pages on the subject, cited by title and section):
 *   - "会议长序列建模状态空间模型加速：深度剖析Mamba硬件感知算子融合与选择性扫描并行化策略"
 *     (ufo.work) §1.1: the recurrence with Abar = exp(Delta A), Bbar = Delta B, y = C h and
 *     input-dependent Delta, B, C; §3.1: chunk transfer operators composed across chunks;
 *     §4.1: a persistent state pool and a one-token update kernel; §4.2: packed sequences with
 *     cu_seqlens and a state reset at each boundary.
 *   - "企业官网建设流程全解析" (discosf.com) §1.1: the skip term y = C h + D x; §1.2: the
 *     zero-order-hold discretisation; §1.3: Delta = softplus of a per-token linear map (here:
 *     delta + per-channel bias).
 *   The pages do not fix the bias placement or the output gate; this library puts the bias
 *   inside the softplus and multiplies the whole output by silu(z) = z * sigmoid(z) when z is
 *   given.  The gated value never feeds back into the state.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library never
 *     allocates device memory and never synchronises the stream (except
 *     ssm_get_device_status, which must read a device word back).
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default).
 *   - Errors are returned as ssm_status_t; nothing is thrown.  Argument checks on the host
 *     happen before any launch: on error nothing is launched and outputs are untouched.
 *     Problems found by a kernel (e.g. an out-of-range slot id) are recorded in a device
 *     status word read by ssm_get_device_status.
 *   - Host threads: every entry point may be called from several host threads at once, on
 *     the same device or on different ones (one thread per GPU is the intended use).  The
 *     only host state is a table of per-(kernel, device) launch facts, filled on first use
 *     under a lock, and the lock-guarded no-allocation scratch (ssm_scan_fwd_noalloc).
 *     Concurrent calls must not share a workspace or outputs.
 *   - Element strides are in elements; the time axis always has stride 1.  A stride of 0
 *     means "contiguous" (the natural value for the documented layout).
 *   - Inputs u, delta, z, B, C have the dtype `dtype`; y has it too unless y_fp32 is set
 *     (then y is float32).  A, Dskip, delta_bias and all states (h0, h_last, the decode pool)
 *     are float32.  Arithmetic is float32; a bf16 y is rounded to nearest-even once, at the
 *     store.
 *   - Supported state sizes: dstate in {16, 32, 64, 128, 256} for the scans, any multiple of
 *     4 up to 256 for the decode update.  Other values return SSM_ERR_UNSUPPORTED.
 *   - Fast path: when every tensor base is 16-byte aligned and every row stride is a
 *     multiple of 16 bytes, inputs are staged with TMA bulk copies, and rows are read up to
 *     the sequence length rounded up to 16 bytes (the row stride covers it).  Other layouts
 *     are accepted and take a slower element-wise staging path.
 */
#ifndef SSM_SCAN_H_
#define SSM_SCAN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SSM_ABI_VERSION 5

typedef enum {
  SSM_OK = 0,
  SSM_ERR_INVALID_ARG = 1, /* null pointer where one is required, bad size/stride/alignment  */
  SSM_ERR_UNSUPPORTED = 2, /* a valid request the library has no kernel for (e.g. dstate = 24) */
  SSM_ERR_CUDA = 3,        /* a CUDA runtime call failed (launch error, no device, ...)      */
  SSM_ERR_BAD_SLOT = 4,    /* device-detected: a decode slot id outside [0, num_slots)       */
  SSM_ERR_TIMEOUT = 5,     /* device-detected: a bounded wait on another CTA gave up          */
  SSM_ERR_WORKSPACE = 6    /* workspace pointer/size smaller than ssm_scan_workspace_size()   */
} ssm_status_t;

typedef enum { SSM_F32 = 0, SSM_BF16 = 1 } ssm_dtype_t;

/*
 * Discretisation of the input matrix (A is diagonal: one value per (channel, state)).
 *   SSM_DISC_EULER: Bbar = Delta B ("会议长序列建模…" page, ufo.work, §1.1); the default.
 *   SSM_DISC_ZOH:   zero-order hold, Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B
 *                   ("企业官网建设流程全解析" page, discosf.com, §1.2), i.e. (exp(Delta A) - 1) / A * B
 *                   per (channel, state), and Delta B where A = 0.
 * Abar = exp(Delta A) in both.
 */
typedef enum { SSM_DISC_EULER = 0, SSM_DISC_ZOH = 1 } ssm_discretization_t;

/*
 * Kernel choice for the prefill scans (ssm_scan_fwd, ssm_scan_fwd_varlen,
 * ssm_scan_fwd_varlen_pool, ssm_scan_fwd_noalloc).  Both compute the same recurrence; they
 * differ in where the parallelism comes from.
 *   SSM_ALGO_AUTO:       the library picks (the default).
 *   SSM_ALGO_CHUNKED:    chunks of every sequence are split into time segments across the
 *                        lanes of a warp and composed with the chunk transfer operators
 *                        (ufo.work page, §3.1); suits few, long sequences.  Every case.
 *   SSM_ALGO_SEQUENTIAL: every lane walks time step by step for one channel and a group of
 *                        its states (no composition); suits many channels x sequences.
 *                        dstate 16 or 32, Euler discretisation, 16-byte aligned rows only;
 *                        other cases return SSM_ERR_UNSUPPORTED.
 * AUTO takes CHUNKED (the faster of the two on every workload measured).  Other values ->
 * SSM_ERR_INVALID_ARG.
 */
typedef enum { SSM_ALGO_AUTO = 0, SSM_ALGO_CHUNKED = 1, SSM_ALGO_SEQUENTIAL = 2 } ssm_algorithm_t;

/* Opaque CUDA stream handle; pass a cudaStream_t (they are the same pointer type). */
typedef struct CUstream_st *ssm_stream_t;

/*
 * Problem description shared by all entry points.
 *
 * Fixed-length batch (ssm_scan_fwd):
 *   u, delta, z, y : [batch][dim][seqlen]   element (b,d,t) at b*x_batch_stride + d*x_dim_stride + t
 *   B, C           : [batch][dstate][seqlen] element (b,n,t) at b*bc_batch_stride + n*bc_state_stride + t
 *   A              : [dim][dstate] contiguous; Dskip, delta_bias : [dim]
 *   h0, h_last     : [batch][dim][dstate] contiguous
 * Packed varlen (ssm_scan_fwd_varlen): batch = 1 and seqlen = total tokens T; sequences are
 *   the column ranges [cu_seqlens[i], cu_seqlens[i+1]) of u, delta, z, y ([dim][T], row
 *   stride x_dim_stride >= T) and of B, C ([dstate][T], row stride bc_state_stride >= T);
 *   h0, h_last : [nseq][dim][dstate].
 * Decode (ssm_state_update): batch = R requests, seqlen = 1; u, delta, z, y : [R][dim] with row
 *   stride x_batch_stride (>= dim); B, C : [R][dstate] with row stride bc_batch_stride.
 *
 * Optional pointers (may be NULL): z (no gate), Dskip (= 0), delta_bias (= 0), h0 (zero
 * state), h_last (final state not written).  Required: u, delta, B, C, A, y.
 *
 * Channel groups (scans only; ufo.work page §3.2 splits channels into independent groups):
 *   with ngroups = G > 1, dim must be a multiple of G and channel d reads B and C of group
 *   d / (dim / G): B, C become [batch][G][dstate][seqlen] (varlen: [G][dstate][T]) with the
 *   group stride bc_group_stride (default dstate * bc_state_stride; the default batch
 *   stride becomes G * dstate * bc_state_stride).  ssm_state_update takes ngroups <= 1 only.
 */
typedef struct ssm_scan_params {
  ssm_dtype_t dtype;       /* dtype of u, delta, z, B, C (and of y unless y_fp32 is set)       */
  int32_t y_fp32;          /* nonzero: y is written as float32 whatever `dtype` is             */
  int64_t batch;
  int64_t dim;
  int64_t dstate;
  int64_t seqlen;
  int64_t x_batch_stride;  /* 0 -> dim * x_dim_stride (batch mode); dim (decode)            */
  int64_t x_dim_stride;    /* 0 -> seqlen                                                    */
  int64_t bc_batch_stride; /* 0 -> dstate * bc_state_stride (batch mode); dstate (decode)    */
  int64_t bc_state_stride; /* 0 -> seqlen                                                    */
  const void *u;
  const void *delta;
  const void *z;
  const void *B;
  const void *C;
  const float *A;
  const float *Dskip;
  const float *delta_bias;
  const float *h0;
  void *y;
  float *h_last;
  int64_t ngroups;         /* channel groups with their own B, C: 0 or 1 = one group (scans)    */
  int64_t bc_group_stride; /* 0 -> dstate * bc_state_stride                                    */
  int32_t discretization;  /* ssm_discretization_t; other values -> SSM_ERR_INVALID_ARG (all calls) */
  int32_t algorithm;       /* ssm_algorithm_t (prefill scans; ignored by ssm_state_update)        */
} ssm_scan_params;

/*
 * Fixed-length batched prefill scan (ufo.work page §1.1 recurrence, §3.1 chunked carry).
 * `workspace` may be NULL when ssm_scan_workspace_size() returns 0; otherwise it must point
 * to that many bytes of device memory that no concurrent call uses.  Its contents on entry
 * do not matter.
 */
ssm_status_t ssm_scan_fwd(const ssm_scan_params *p, void *workspace, size_t workspace_bytes,
                          ssm_stream_t stream);

/*
 * Packed variable-length scan (ufo.work page §4.2): `cu_seqlens` is a DEVICE int32 array of
 * nseq+1 non-decreasing offsets with cu_seqlens[0] = 0 and cu_seqlens[nseq] = p->seqlen.
 * Each sequence starts from h0[i] (or zero) and h_last[i] receives its final state; empty
 * sequences produce h_last[i] = h0[i] (or zero).  The offsets are read on the device only.
 */
ssm_status_t ssm_scan_fwd_varlen(const ssm_scan_params *p, const int32_t *cu_seqlens, int64_t nseq,
                                 void *workspace, size_t workspace_bytes, ssm_stream_t stream);

/*
 * Packed prefill into a slot-indexed state pool (ufo.work second article §4.2, chunked
 * prefill; §4.1 state pool): the same scan as ssm_scan_fwd_varlen, but sequence i starts
 * from pool[slot_ids[i]] and its final state is written back there, so a long prompt can be
 * fed in pieces over several calls and then decoded with ssm_state_update on the same pool.
 *   pool     : DEVICE float32 [num_slots][dim][dstate], read and written in place
 *   slot_ids : DEVICE int32 [nseq]; ids must be distinct (duplicates race).  An id outside
 *              [0, num_slots) starts that sequence from zero, leaves the pool untouched (y is
 *              still written) and records SSM_ERR_BAD_SLOT in the device status word.
 * p->h0 and p->h_last must be NULL (SSM_ERR_INVALID_ARG otherwise).  Workspace as for
 * ssm_scan_fwd_varlen (ssm_scan_workspace_size with the same nseq).
 */
ssm_status_t ssm_scan_fwd_varlen_pool(const ssm_scan_params *p, const int32_t *cu_seqlens, int64_t nseq,
                                      float *pool, int64_t num_slots, const int32_t *slot_ids,
                                      void *workspace, size_t workspace_bytes, ssm_stream_t stream);

/*
 * One decode step over a slot-indexed state pool (ufo.work page §4.1 and its second
 * article §4.1): for each request r, h = pool[slot_ids[r]] ([dim][dstate] float32) advances
 * by one token in place and y[r] is written.  `slot_ids` is a DEVICE int32 array of R ids;
 * ids must be distinct (duplicates race).  An id outside [0, num_slots) is skipped (its y row
 * is not written) and SSM_ERR_BAD_SLOT is recorded in the device status word.
 * p->batch must equal R and p->seqlen must be 1; p->h0 and p->h_last are ignored.
 */
ssm_status_t ssm_state_update(float *pool, int64_t num_slots, const int32_t *slot_ids, int64_t R,
                              const ssm_scan_params *p, ssm_stream_t stream);

/*
 * Gradients of the fixed-length batch scan: the reverse-mode derivative of ssm_scan_fwd's
 * outputs y and h_last with respect to u, delta, z, B, C, A, Dskip, delta_bias and h0, for
 * training.  It follows the schedule of the "会议长序列建模…" page (ufo.work), §2.2 (strategy B:
 * keep checkpoints, recompute the rest) and its second article, §3.1 (chunk-boundary states
 * and the composition of chunk operators): the sequence is cut into time segments; a first
 * pass keeps, per segment, its state every 8 steps from a zero start and its zero-start
 * forward and adjoint operators (in the workspace); the operators are composed across the
 * segments (the true state entering and adjoint leaving each); then every segment is walked
 * backwards, each 8-step stretch recomputed from its checkpoint and the adjoint recurrence
 * dh_{t-1} = exp(Delta_t A) (dh_t + C_t dyraw_t) carried from the segment's end.  dA, dDskip,
 * ddelta_bias, dB and dC are sums formed with atomics, so their last bits may differ from
 * call to call; du, ddelta, dz and dh0 are reproducible.
 *
 * `p` describes the forward problem as for ssm_scan_fwd (the same inputs; p->y and p->h_last
 * are not used and may be NULL).  Supported:
 * dstate 16, ngroups <= 1, either discretisation (Euler or the zero-order hold, whose input
 * coefficient c = (exp(Delta A) - 1) / A has dc/dDelta = exp(Delta A) and
 * dc/dA = (Delta exp(Delta A) - c) / A), and every tensor base and row stride 16-byte aligned
 * (the forward's fast path; dy, du, ddelta and dz included).  Other cases return
 * SSM_ERR_UNSUPPORTED before anything runs.
 *
 * Every gradient is overwritten (not accumulated into).  "The dtype of y" below is the input
 * dtype, or float32 when p->y_fp32 is set.
 *   dy          : [batch][dim][seqlen] in the dtype of y, strides as u (required)
 *   dh_last     : [batch][dim][dstate] float32, gradient of h_last, or NULL (zero)
 *   du, ddelta  : [batch][dim][seqlen] in the dtype of y, strides as u (required)
 *   dz          : the same; required when p->z is given, ignored otherwise
 *   dB, dC      : [batch][dstate][seqlen] float32, contiguous (required)
 *   dA          : [dim][dstate] float32 (required)
 *   dDskip, ddelta_bias : [dim] float32, or NULL (not computed)
 *   dh0         : [batch][dim][dstate] float32, or NULL (not computed)
 * The workspace (ssm_scan_bwd_workspace_size bytes, 16-byte aligned) holds the checkpoints
 * and the per-segment operators; its contents on entry do not matter.
 */
typedef struct ssm_scan_grads {
  const void *dy;
  const float *dh_last;
  void *du;
  void *ddelta;
  void *dz;
  float *dB;
  float *dC;
  float *dA;
  float *dDskip;
  float *ddelta_bias;
  float *dh0;
} ssm_scan_grads;
ssm_status_t ssm_scan_bwd(const ssm_scan_params *p, const ssm_scan_grads *g, void *workspace,
                          size_t workspace_bytes, ssm_stream_t stream);

/* Bytes of device workspace ssm_scan_bwd needs for this problem (0 if it is not supported). */
size_t ssm_scan_bwd_workspace_size(const ssm_scan_params *p);

/*
 * SSD (Mamba-2) chunked form of the scan on the tensor cores: the second article of the
 * "会议长序列建模…" page (ufo.work), "Mamba-2/SSD架构下的矩阵化加速范式…", §1.1 (the scan as masked
 * attention, Y = (mask o (C B^T)) V with V = Delta x) and §2.2 (the mask carries the decay
 * exp(A sum Delta) from a prefix sum), with the state carried between chunks.  A is one scalar
 * per head and Delta one value per (head, step), shared by the head's headdim channels; B and C
 * are shared by all heads.  For head h, channel p and state n:
 *     h_t[p][n] = exp(dt[h][t] A[h]) h_{t-1}[p][n] + dt[h][t] B[n][t] x[h][p][t]
 *     y[h][p][t] = sum_n C[n][t] h_t[p][n]
 * -- the selective scan with A[d][n] = A[h] for the channels d of head h and Delta given
 * directly (no softplus, no skip term, no gate).  Computed in chunks of 128 steps as four
 * dense products per chunk on tcgen05 (float16 operands, float32 accumulation).
 *   x      : DEVICE bf16 [batch][nheads][headdim][seqlen]
 *   dt     : DEVICE float32 [batch][nheads][seqlen], the step Delta (> 0)
 *   A      : DEVICE float32 [nheads] (< 0 for a decaying state)
 *   B, C   : DEVICE bf16 [batch][dstate][seqlen]
 *   h0     : DEVICE float32 [batch][nheads][headdim][dstate] or NULL (zero)
 *   y      : DEVICE bf16 [batch][nheads][headdim][seqlen] (written)
 *   h_last : DEVICE float32 [batch][nheads][headdim][dstate] or NULL (not written)
 * Supported: headdim 64, dstate 128, seqlen a multiple of 8, 16-byte aligned x, B, C;
 * SSM_ERR_UNSUPPORTED otherwise.  Contiguous tensors.  No workspace.
 */
typedef struct ssm_ssd_params {
  int64_t batch;
  int64_t nheads;
  int64_t headdim;
  int64_t dstate;
  int64_t seqlen;
  const void *x;
  const float *dt;
  const float *A;
  const void *B;
  const void *C;
  const float *h0;
  void *y;
  float *h_last;
} ssm_ssd_params;
ssm_status_t ssm_ssd_fwd(const ssm_ssd_params *p, ssm_stream_t stream);

/*
 * Allocation-free variant of ssm_scan_fwd.  (The pages have no counterpart; this is a
 * library convenience.)
 *
 * Some callers cannot allocate device memory while they run: a plugin inside an inference
 * engine whose enqueue step must not allocate, or a serving loop that bans cudaMalloc after
 * start-up because cudaMalloc can synchronise the device and stall other streams.  Such a
 * caller cannot provide the workspace ssm_scan_fwd may ask for.  This entry point takes the
 * same problem description and computes the same result, but its scratch is a static device
 * array of SSM_NOALLOC_SCRATCH_BYTES inside the library (every GPU that loads the library
 * holds it until the process exits).  It calls no cudaMalloc, cudaFree or other allocating
 * routine.
 *   - The first call on a device looks up the array's device address for that device
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - A problem whose scratch need (ssm_scan_workspace_size) exceeds
 *     SSM_NOALLOC_SCRATCH_BYTES is rejected with SSM_ERR_WORKSPACE before anything runs.
 *   - All calls share the one array and it keeps the last call's contents; each call clears
 *     the part that must start at zero (an asynchronous memset on `stream`).  Calls that can
 *     overlap on the GPU (e.g. on two streams without ordering) race on the array: order them.
 */
#define SSM_NOALLOC_SCRATCH_BYTES (4u << 20)
ssm_status_t ssm_scan_fwd_noalloc(const ssm_scan_params *p, ssm_stream_t stream);

/* Bytes of device workspace the scan entry points need for this problem (0 if none).
 * For the fixed-length scan pass nseq = 0. */
size_t ssm_scan_workspace_size(const ssm_scan_params *p, int64_t nseq);

/* Synchronises `stream`, then reads and clears the device status word (SSM_OK if no kernel
 * reported a problem since the last call). */
ssm_status_t ssm_get_device_status(ssm_stream_t stream);

/* Human-readable name of a status code (static storage). */
const char *ssm_status_string(ssm_status_t s);

/* SSM_ABI_VERSION of the built library. */
int ssm_abi_version(void);

/*
 * TEST HOOK -- not for production use.  The next fixed-length scan that runs on the
 * persistent grid (rows 16-byte aligned, more than one chunk) splits every chain into
 * one-chunk units and starts its unit counter past the first chunk group: no unit of that
 * group runs, so the units after it wait for a hand-off that never comes.  Their wait is
 * bounded; on giving up the kernel records SSM_ERR_TIMEOUT in the status word and finishes
 * with unusable outputs, and the context stays usable.  The hook applies to one launch and
 * then clears itself.  It lets a test show that the hand-off wait cannot hang the GPU.
 */
void ssm_test_drop_first_handoff(void);

#ifdef __cplusplus
}
#endif

#endif /* SSM_SCAN_H_ */
