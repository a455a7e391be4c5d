/*
 * gdn.h -- C ABI of the B200 (sm_100a) Gated DeltaNet chunked-prefill library.
 *
 * The operator (named on the pages "Qwen's FlashQLA targets the expensive bit of
 * long-context AI", section "What happened", and "FlashQLA resource", section 2,
 * row "What it serves": forward and backward of GDN chunked prefill) is the
 * gated delta-rule recurrence, per sequence and value head,
 *
 *     S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = scale * S_t q_t,
 *
 * with S (dv x dk) carried as its transpose h = S^T (dk x dv) in h0 / hT.
 * The library evaluates it chunk-parallel (64-token chunks, WY/UT transform)
 * and, for long sequences with few heads, splits a sequence across SMs
 * ("gate-driven automatic intra-card context parallelism", "FlashQLA resource",
 * section 3, first row of the feature table), stitching segments exactly through
 * their affine state maps h_end = M h_start + b.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller. The library
 *     never allocates device memory; scratch space comes from `workspace`,
 *     whose size the matching *_workspace_size() returns (at least 256 bytes,
 *     256-byte aligned).
 *   - Layouts follow the (batch, seqlen, heads, head_dim) convention with the
 *     last dimension contiguous ("FA4 SM120 bundle" page, API notes on tensor
 *     layout; packed sequences via cu_seqlens, same page, "Variable-length"):
 *       q, k  [B, T, Hqk, dk]      v, o, dO  [B, T, Hv, dv]
 *       g, beta, dg, dbeta [B, T, Hv]
 *       h0, hT, dhT, dh0 [N, Hv, dk, dv] fp32, N = B (or num_seqs when packed)
 *     All arrays are dense and contiguous; base pointers 16-byte aligned.
 *   - Grouped values: Hv must be a multiple of Hqk; v-head j reads q/k head
 *     j / (Hv / Hqk). dq / dk of a q/k head sum over the v-heads that read it.
 *   - Packed variable-length input: cu_seqlens (device int32 [num_seqs + 1],
 *     0 = cu[0] <= cu[1] <= ... <= cu[num_seqs] = T) requires B == 1. Sequences
 *     never interact. Chunks restart at every sequence start.
 *   - dtype: GDN_BF16 = q, k, v, beta, o, dO, dq, dk, dv, dbeta in bfloat16;
 *     GDN_F32 = those in fp32. g, dg, h0, hT, dhT, dh0 are always fp32.
 *     Internal state and accumulation are fp32 in both cases.
 *   - dk, dv in {64, 128}; bf16 with dk = dv = 128 runs the tensor-core
 *     (tcgen05/TMEM/TMA) kernels; every other supported case runs the fp32
 *     CUDA-core kernels. Anything else returns GDN_ERR_UNSUPPORTED.
 *   - Calls are asynchronous on `stream` and never synchronise. Arguments are
 *     validated on the host before anything is launched; an invalid call
 *     returns an error status and touches no output. Errors a kernel detects
 *     (an inconsistent cu_seqlens, a bounded wait that timed out) are recorded
 *     in the workspace's status word, reported by gdn_read_device_status(), and
 *     in a per-device word, reported by gdn_check_device_error(). Outputs of a
 *     call whose kernels recorded an error are unspecified.
 *   - Launch failures return GDN_ERR_CUDA.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = 1,     /* bad shape, null required pointer, misaligned pointer, bad cu_seqlens */
  GDN_ERR_UNSUPPORTED = 2,     /* valid but not implemented (e.g. dk = 96)                             */
  GDN_ERR_WORKSPACE = 3,       /* workspace null, too small or misaligned                              */
  GDN_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed                                 */
  GDN_ERR_DEVICE_TIMEOUT = 5,  /* a kernel's bounded wait gave up (reported via the status word)       */
  GDN_ERR_DEVICE_INPUT = 6,    /* a kernel found device-side input inconsistent (cu_seqlens)          */
  GDN_ERR_DEVICE_LAUNCH = 7    /* a kernel found its launch unusable (dynamic shared memory misaligned) */
} gdn_status;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

/* Optional knobs; pass NULL for the defaults (all zero). */
typedef struct {
  /* Intra-card context parallelism on the tensor-core path ("FlashQLA resource", section 3,
   * "Gate-driven automatic intra-card context parallelism"):
   *   0 = automatic: sequences are split into segments when (sequences x v-heads) leaves SMs
   *       idle; -1 = off; n > 0 = at most n segments per sequence, each of ceil(ceil(T / 64) / n)
   *       chunks (T = B's sequence length, or the packed total). */
  int cp_mode;
  /* 0 or 1 (anything else: GDN_ERR_INVALID_ARG). Every kernel of this library reduces in a
   * fixed order (no floating-point atomics, fixed per-producer slots), so results are
   * bit-reproducible from run to run whatever the value; 1 is accepted for callers that ask
   * for determinism explicitly and changes nothing. */
  int deterministic;
  /* Finer control of the segment length, overriding cp_mode when nonzero: n > 0 = segments
   * of n chunks (64 tokens each), -1 = off. */
  int cp_segment_chunks;
  /* How a segment obtains its start state (0, 1 or 2; anything else GDN_ERR_INVALID_ARG).
   * Gate-driven start: the segment's CTA runs, from a zero state, the shortest window of
   *   preceding chunks whose transition has spectral norm <= 2^-64 (each token's factor
   *   exp(g) max(1, |1 - beta |k|^2|) is exact), so the dropped part is below fp32
   *   resolution. The backward's reverse chain does the same after a segment's end.
   * Exact affine stitch: phase 1 computes a segment's map h_end = M h_start + b, phase 2
   *   chains the maps, phase 3 reruns the segment from its stitched start state. The backward
   *   mirrors it on the state gradient, dh_start = M' dh_end + c, chained from the sequence end.
   * 0 (default): gate-driven; a segment without such a window within 16 chunks (weakly
   *   decaying heads) restarts at the sequence start (the plain recurrence). The smallest
   *   workspace: no per-segment maps.
   * 1: the exact stitch for every segment.
   * 2: gate-driven, with the exact stitch for the segments whose window does not close, once a
   *   sequence can have 3 or more segments (with 2, as 0). A probe kernel records every
   *   segment's window first and phase 1 maps only the segments that need it; the two extra
   *   launches and phase 1's grid cost tens of microseconds even when every window closes, so
   *   this pays off for long sequences with weakly decaying heads. */
  int cp_exact;
  /* Chunk start states cached between a forward and its backward (tensor-core path:
   * bf16, dk = dv = 128), device memory of gdn_chunk_states_size() bytes, 16-byte
   * aligned, owned by the caller. NULL (default): nothing is cached and the backward
   * recomputes the states itself.
   *   gdn_chunk_fwd writes, for every chunk c of every sequence n and v-head j, the
   *     state at the chunk's first token in bf16, transposed: states[slot][j][r][d] =
   *     h[d][r] (r < dv, d < dk), slot = n * ceil(T/64) + c for independent sequences,
   *     or (sum over m < n of ceil(len_m / 64)) + c for packed ones; after all slots, the
   *     chunk's A = (I + L)^-1 (fp32, 64 x 64 row-major), then its P = lower_incl(Q K^T * E)
   *     (bf16, 64 x 64, 128-byte-swizzled rows), both in the same slot order.
   *   gdn_chunk_bwd reads them instead of running its forward pass; they must come
   *     from gdn_chunk_fwd on the same q, k, v, g, beta, h0, cu_seqlens and qk_l2norm.
   * Set on another path: GDN_ERR_UNSUPPORTED; not 16-byte aligned: GDN_ERR_INVALID_ARG. */
  void* states;
  /* 1: every q and k row is L2-normalised inside the kernels, x / sqrt(|x|^2 + 1e-6), and the
   * backward returns the gradients with respect to the raw (unnormalised) q and k. 0: q and k
   * are used as given. Tensor-core path only (bf16, dk = dv = 128); elsewhere
   * GDN_ERR_UNSUPPORTED. */
  int qk_l2norm;
  /* Testing only; must be 0 in production. 1: every CTA of the forward's tensor-core kernel
   * first waits on a barrier that nothing completes; the wait gives up after about 1 ms and
   * records GDN_ERR_DEVICE_TIMEOUT (in the workspace's status word and the per-device word),
   * then the call completes its work as usual. It lets a test see a bounded wait run out
   * without faulting or hanging the GPU. */
  int test_stall;
  /* Reserved, must be 0. */
  int reserved[2];
} gdn_options;

/* Bytes of the chunk-state cache (gdn_options.states) for these sizes. */
size_t gdn_chunk_states_size(int B, int T, int Hqk, int Hv, int dk, int dv, int num_seqs);

/* Bytes of device workspace gdn_chunk_fwd needs for these sizes and options. */
size_t gdn_chunk_fwd_workspace_size(int B, int T, int Hqk, int Hv, int dk, int dv,
                                    int num_seqs, const gdn_options* opt);

/*
 * Forward. Computes o [B,T,Hv,dv] (dtype) and, if hT != NULL, the final state
 * of every (sequence, v-head) in hT [N,Hv,dk,dv] fp32.
 *   q, k, v, beta : dtype;  g : fp32 raw per-token log-decay (<= 0 in GDN,
 *                   not required); scale : multiplies S_t q_t (usually dk^-0.5)
 *   h0            : nullable, [N,Hv,dk,dv] fp32 (NULL = zero initial state)
 *   cu_seqlens    : nullable device int32 [num_seqs+1] (NULL = B independent
 *                   sequences of length T; num_seqs is then ignored)
 *   workspace     : device scratch of >= gdn_chunk_fwd_workspace_size() bytes
 */
gdn_status gdn_chunk_fwd(gdn_dtype dtype, int B, int T, int Hqk, int Hv, int dk, int dv,
                         const void* q, const void* k, const void* v,
                         const float* g, const void* beta, float scale,
                         const float* h0, const int32_t* cu_seqlens, int num_seqs,
                         void* o, float* hT,
                         void* workspace, size_t workspace_bytes,
                         const gdn_options* opt, cudaStream_t stream);

/* Bytes of device workspace gdn_chunk_bwd needs for these sizes and options. */
size_t gdn_chunk_bwd_workspace_size(int B, int T, int Hqk, int Hv, int dk, int dv,
                                    int num_seqs, const gdn_options* opt);

/*
 * Backward ("FlashQLA resource", section 5: backward and its intra-card
 * sequence parallelism). Given the forward inputs and the incoming gradients
 * dO [B,T,Hv,dv] (dtype) and dhT (nullable, [N,Hv,dk,dv] fp32), writes
 *   dq, dk [B,T,Hqk,dk] (dtype; summed over the v-heads sharing a q/k head),
 *   dv [B,T,Hv,dv] (dtype), dg [B,T,Hv] fp32 (w.r.t. the raw per-token g),
 *   dbeta [B,T,Hv] (dtype), dh0 (nullable) [N,Hv,dk,dv] fp32.
 * Unless opt->states holds the chunk start states of the matching forward call
 * (see gdn_options.states), the forward pass is recomputed inside the call.
 * bf16 with dk = dv = 128 runs on tensor cores. The other supported sizes (fp32, or a head
 * dim of 64) run the exact token-level adjoint on CUDA cores, one (sequence, v-head) per CTA
 * with the states recomputed from fp32 checkpoints every 64 tokens; that path takes neither
 * opt->states nor opt->qk_l2norm (GDN_ERR_UNSUPPORTED).
 */
gdn_status gdn_chunk_bwd(gdn_dtype dtype, int B, int T, int Hqk, int Hv, int dk, int dv,
                         const void* q, const void* k, const void* v,
                         const float* g, const void* beta, float scale,
                         const float* h0, const int32_t* cu_seqlens, int num_seqs,
                         const void* dO, const float* dhT,
                         void* dq, void* dk_out, void* dv_out, float* dg, void* dbeta,
                         float* dh0,
                         void* workspace, size_t workspace_bytes,
                         const gdn_options* opt, cudaStream_t stream);

/*
 * One recurrent (decode) step per sequence and v-head, continuing a prefill: with
 * h = S^T the current state (for instance the hT of gdn_chunk_fwd),
 *     h <- exp(g) h;   r = v - h^T k;   h <- h + beta k r^T;   o = scale h^T q,
 * i.e. the recurrence above for a single token. The pages list on-device agentic
 * inference among the scenarios ("FlashQLA resource", section 4, table of the
 * authors' stated results); generation after a prefill runs this step.
 *   q, k  [N, Hqk, dk] (dtype)     v, o [N, Hv, dv] (dtype)
 *   g     [N, Hv] fp32 (raw log-decay)   beta [N, Hv] (dtype)
 *   state [N, Hv, dk, dv] fp32, read and overwritten in place (the caller's h0/hT
 *         layout); it must not overlap the other arrays.
 * dk, dv in {64, 128, 256} (any pair); dtype GDN_BF16 or GDN_F32 (fp32 arithmetic in both).
 * N = 0 is a no-op. Null or misaligned pointers, Hv not a multiple of Hqk:
 * GDN_ERR_INVALID_ARG; other head dims or N * Hv * dv / 64 >= 2^31: GDN_ERR_UNSUPPORTED;
 * launch failure: GDN_ERR_CUDA. Asynchronous on `stream`; needs no workspace.
 */
gdn_status gdn_recurrent_step(gdn_dtype dtype, int N, int Hqk, int Hv, int dk, int dv,
                              const void* q, const void* k, const void* v,
                              const float* g, const void* beta, float scale,
                              float* state, void* o, cudaStream_t stream);

/*
 * Forward without a workspace, for callers that cannot allocate device memory where
 * they run the operator (inside a framework's memory pool, or a runtime that forbids
 * allocation on its hot path). The pages have no counterpart: this is a library
 * convenience, not part of the method.
 *
 * Same arguments and results as gdn_chunk_fwd, minus the workspace. Scratch comes from
 * a 1 MiB array in the library's device memory that every GPU loading the library holds
 * until the process exits; the call allocates nothing (no cudaMalloc, no library
 * allocator). Calls whose scratch need (gdn_chunk_fwd_workspace_size) exceeds 1 MiB,
 * e.g. the exact affine stitch (cp_exact) on large inputs, return GDN_ERR_WORKSPACE
 * with the sizes in gdn_last_error(). With cp_exact = 2 and too little room for its
 * per-segment maps, the call uses cp_exact = 0 (segments without a closing window restart
 * at the sequence start). The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress, once per device); make that first call before
 * any stream capture. The address is kept for the life of the process: after a
 * cudaDeviceReset the array is reloaded elsewhere, so do not use this entry point on a
 * device that was reset. All calls share the one array: calls that overlap on the GPU
 * (concurrent streams) race and must not be issued. Each call clears the status word;
 * device-side findings (inconsistent cu_seqlens, a timed-out wait) are not reported
 * back through this entry point.
 */
gdn_status gdn_chunk_fwd_noalloc(gdn_dtype dtype, int B, int T, int Hqk, int Hv, int dk, int dv,
                                 const void* q, const void* k, const void* v,
                                 const float* g, const void* beta, float scale,
                                 const float* h0, const int32_t* cu_seqlens, int num_seqs,
                                 void* o, float* hT,
                                 const gdn_options* opt, cudaStream_t stream);

/*
 * Host-buffer calls: the forward and/or the backward on arrays in host memory, for callers
 * whose data is not on the GPU (the pages' scenarios include on-device agentic inference,
 * "FlashQLA resource", section 4). Every input is copied to the device, the same kernels as
 * gdn_chunk_fwd / gdn_chunk_bwd run, and every output is copied back; the call enqueues all of
 * it and returns (asynchronous to the calling thread).
 *   mode GDN_HOST_FWD:     q k v g beta [h0] [cu_seqlens] -> o [hT]
 *   mode GDN_HOST_BWD:     q k v g beta [h0] [cu_seqlens] dO [dhT] -> dq dk dv dg dbeta [dh0]
 *                          (the forward pass is recomputed inside)
 *   mode GDN_HOST_FWD_BWD: both; on the tensor-core sizes (bf16, dk = dv = 128) the backward
 *                          reads the forward's chunk-state cache, which lives in the scratch, and
 *                          on the others it recomputes the forward pass.
 * Arrays, shapes, dtypes and limits as in gdn_chunk_fwd / gdn_chunk_bwd; bracketed ones are
 * nullable, unused ones are ignored. Host arrays need no alignment; page-locked memory
 * (cudaHostAlloc, cudaHostRegister) lets the copies run asynchronously and overlap, pageable
 * memory works but every copy then blocks the thread.
 *   scratch  device memory of >= gdn_chunk_host_scratch_size() bytes, 256-byte aligned, owned
 *            by the caller: the device copies of all arrays, the cache and the workspaces.
 *   stream   the kernels.  h2d_stream / d2h_stream: the input / output copies (NULL: stream).
 *            With three distinct streams and two scratch buffers used in turn, one call's
 *            outputs go back while the next call's inputs come in.
 * Ordering: a call's input copies wait for the kernels of the previous call on the same
 * scratch, and its kernels wait for that call's output copies (the library keeps a few CUDA
 * events per scratch address, created on its first use on the current device; beyond 64
 * addresses, those whose recorded work has completed are released). The outputs are
 * in host memory once d2h_stream (or stream) has passed the call. opt->states must be NULL
 * (GDN_ERR_INVALID_ARG). Device-side findings go to the per-device status word
 * (gdn_check_device_error). A failing CUDA call returns GDN_ERR_CUDA; copies already enqueued
 * then still run.
 */
typedef enum { GDN_HOST_FWD = 1, GDN_HOST_BWD = 2, GDN_HOST_FWD_BWD = 3 } gdn_host_mode;

/* Bytes of scratch gdn_chunk_host needs (0 for invalid sizes). With B == 1 and num_seqs >= 1 it
 * covers both a packed call and a call without cu_seqlens. */
size_t gdn_chunk_host_scratch_size(gdn_host_mode mode, gdn_dtype dtype, int B, int T, int Hqk, int Hv,
                                   int dk, int dv, int num_seqs, const gdn_options* opt);

gdn_status gdn_chunk_host(gdn_host_mode mode, gdn_dtype dtype, int B, int T, int Hqk, int Hv, int dk, int dv,
                          const void* q, const void* k, const void* v,
                          const float* g, const void* beta, float scale,
                          const float* h0, const int32_t* cu_seqlens, int num_seqs,
                          const void* dO, const float* dhT,
                          void* o, float* hT,
                          void* dq, void* dk_out, void* dv_out, float* dg, void* dbeta, float* dh0,
                          void* scratch, size_t scratch_bytes, const gdn_options* opt,
                          cudaStream_t stream, cudaStream_t h2d_stream, cudaStream_t d2h_stream);

/* Synchronises `stream`, then returns (and clears) the status word that the
 * kernels of earlier calls on this workspace recorded: GDN_OK,
 * GDN_ERR_DEVICE_TIMEOUT, GDN_ERR_DEVICE_INPUT or GDN_ERR_DEVICE_LAUNCH.
 * GDN_ERR_CUDA if the stream itself reports an error. */
gdn_status gdn_read_device_status(void* workspace, cudaStream_t stream);

/* Synchronises `stream`, then returns (and clears) the library's status word of the current
 * device: the first device-side finding (GDN_ERR_DEVICE_TIMEOUT, GDN_ERR_DEVICE_INPUT,
 * GDN_ERR_DEVICE_LAUNCH) of any gdn_chunk_fwd / gdn_chunk_bwd / gdn_chunk_fwd_noalloc call on
 * this device since the last check, whatever its workspace; GDN_OK if none. The word is found
 * with cudaGetSymbolAddress on every call; a call that cannot find it (for instance the very
 * first library call of a process made under stream capture) records only in its workspace.
 * GDN_ERR_CUDA if the stream or a copy fails (detail in gdn_last_error()). */
gdn_status gdn_check_device_error(cudaStream_t stream);

/* Static, human-readable text of a status code. */
const char* gdn_status_string(gdn_status s);

/* Detail of the last GDN_ERR_CUDA returned on the calling host thread (which call
 * failed and the CUDA error text); empty if none. Static storage, not to be freed. */
const char* gdn_last_error(void);

/*
 * Instrumentation (host-thread local). gdn_trace_begin() creates 2 * capacity
 * timing events; while the trace is active every kernel the library launches
 * from this thread is bracketed by cudaEventRecord on its launch stream (launches
 * beyond `capacity` are not recorded). gdn_trace_end() waits for the recorded
 * events, writes each launch's device time in milliseconds to ms[i] and its kernel
 * id to kernel_ids[i] (both nullable, capacity entries), destroys the events and
 * returns the number of launches recorded (-1 on a CUDA error).
 * gdn_kernel_name() names a kernel id; gdn_launch_count() counts every kernel
 * launched from this thread since the library was loaded.
 */
gdn_status gdn_trace_begin(int capacity);
int gdn_trace_end(float* ms, int* kernel_ids);
const char* gdn_kernel_name(int kernel_id);
long long gdn_launch_count(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
