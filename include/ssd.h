/*
 * ssd.h - C ABI of libssd, the forward pass of the state space dual (SSD) layer
 * on NVIDIA B200 (sm_100a).
 *
 * The layer ("Transformers are SSMs: Generalized Models and Efficient
 * Algorithms Through Structured State Space Duality", Knowl 1) is the
 * scalar-identity selective SSM, per batch row b and head h:
 *
 *     h_t = exp(dt_t * A_h) * h_{t-1} + dt_t * x_t (outer) B_t      h_{-1} = h_init or 0
 *     y_t = C_t . h_t + D_h * x_t
 *
 * evaluated through its dual form Y = (L o C B^T) X with the 1-semiseparable
 * decay mask L_ji = prod_{s=i+1}^{j} a_s, by the block-decomposition algorithm
 * of Knowl 2: chunks of Q tokens, a quadratic (masked attention) product inside
 * each chunk and a linear recurrence over chunk states between chunks.
 *
 * Shapes (row-major, contiguous, innermost last):
 *     x, y            [batch, seqlen, nheads, headdim]      dtype (fp32 or bf16)
 *     dt              [batch, seqlen, nheads]               fp32
 *     A, D            [nheads]                              fp32
 *     B, C            [batch, seqlen, ngroups, dstate]      dtype
 *     states          [batch, nheads, headdim, dstate]      fp32
 * Head h reads B and C of group g = h / (nheads / ngroups) (Knowl 7: grouped
 * heads share B and C; ngroups = 1 is the multi-input pattern).
 *
 * Conventions for every entry point:
 *   - Device pointers are CUDA device (or managed) memory owned by the caller.
 *     The library allocates no device memory and keeps no state between calls,
 *     so calls on different streams or host threads are independent.
 *   - All argument checks run on the host before anything is enqueued; a
 *     rejected call enqueues nothing and returns SSD_ERR_INVALID_ARG or
 *     SSD_ERR_UNSUPPORTED synchronously.
 *   - Device entry points are asynchronous on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream) and never synchronize. A launch failure
 *     returns SSD_ERR_CUDA; ssd_last_error_detail() then names the CUDA error.
 *   - Inputs may alias one another; an output must not overlap any input, any
 *     other output or the workspace (SSD_ERR_INVALID_ARG).
 *   - x, B, C, y, the state tensors and the workspace must be 16-byte aligned;
 *     dt, A and D 4-byte aligned.
 */
#ifndef SSD_H_
#define SSD_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, overlap, small workspace */
    SSD_ERR_UNSUPPORTED = 2,   /* valid shape outside what the kernels implement */
    SSD_ERR_CUDA = 3,          /* a CUDA call failed; see ssd_last_error_detail() */
    SSD_ERR_TIMEOUT = 4        /* a bounded device-side wait gave up */
} ssd_status_t;

typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype_t;

typedef struct {
    int64_t batch;       /* b >= 0                                          */
    int64_t seqlen;      /* T >= 0; T need not be a multiple of chunk_size  */
    int64_t nheads;      /* H >= 1                                          */
    int64_t headdim;     /* P in [1, 256]                                   */
    int64_t ngroups;     /* G >= 1, divides H                               */
    int64_t dstate;      /* N in [1, 256]                                   */
    int64_t chunk_size;  /* Q in {16, 32, 64, 128, 256}                     */
    int32_t dtype;       /* ssd_dtype_t of x, B, C and y                    */
    int32_t reserved;    /* must be 0                                       */
} ssd_shape_t;

/* Human-readable name of a status code (static string, never NULL). */
SSD_API const char* ssd_status_string(ssd_status_t status);

/* Detail of the last SSD_ERR_CUDA / SSD_ERR_TIMEOUT on the calling host thread
 * ("" if none). The pointer stays valid until the next call on that thread. */
SSD_API const char* ssd_last_error_detail(void);

/* Library version as major*10000 + minor*100 + patch. */
SSD_API int ssd_version(void);

/* Which kernels ssd_fwd launches for `shape` (host-only query, nothing runs):
 * *path receives a static name ("fused": one tensor-core kernel per call;
 * "steps": the four step kernels on tensor cores; "simt": the four step kernels
 * on CUDA cores) and *kernels the number of kernel launches per call (the
 * fused path also enqueues one small memset of its workspace counters). */
SSD_API ssd_status_t ssd_fwd_plan(const ssd_shape_t* shape, const char** path, int* kernels);

/* Bytes of device workspace ssd_fwd needs for `shape`, written to *bytes.
 * Returns SSD_ERR_INVALID_ARG / SSD_ERR_UNSUPPORTED for a shape ssd_fwd rejects. */
SSD_API ssd_status_t ssd_fwd_workspace_size(const ssd_shape_t* shape, size_t* bytes);

/*
 * Full SSD layer forward (Knowl 2, whole algorithm; Knowl 1 for the result).
 *   x, dt, A, B, C     inputs as above (device).
 *   D                  [H] fp32 skip weights, or NULL for D = 0.
 *   initial_states     [b,H,P,N] fp32 state entering the sequence, or NULL for 0.
 *   y                  [b,T,H,P] output in `dtype` (device), rounded to nearest even.
 *   final_states       [b,H,P,N] fp32 state after the last token, or NULL to skip.
 *                      Must not be the same memory as initial_states.
 *   workspace          device scratch of at least ssd_fwd_workspace_size() bytes
 *                      (may be NULL when that size is 0). Its contents on entry
 *                      are ignored; concurrent calls need separate workspaces.
 * Result (y, final_states) equals the recurrence above up to rounding: the
 * decay math and accumulation are fp32 for both dtypes.
 */
SSD_API ssd_status_t ssd_fwd(const ssd_shape_t* shape,
                     const void* x, const float* dt, const float* A,
                     const void* B, const void* C, const float* D,
                     const float* initial_states,
                     void* y, float* final_states,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * ssd_fwd without a caller-provided workspace, for callers that cannot
 * allocate device memory: hosts that own every device allocation and give a
 * library only its input and output buffers, or call paths that cannot afford
 * cudaMalloc's possible device-wide synchronization. The pages describe no
 * such entry point; it is a deployment convenience of this library.
 *   Arguments are those of ssd_fwd minus the workspace. Scratch space comes
 *   from one static device array of 64 MiB that every GPU loading libssd
 *   reserves until the process exits. A shape whose ssd_fwd workspace
 *   (ssd_fwd_workspace_size) exceeds 64 MiB is rejected with
 *   SSD_ERR_UNSUPPORTED before anything is enqueued; ssd_last_error_detail()
 *   then says so. The library allocates nothing on this path.
 *   Every call looks up the current device's copy of the array
 *   (cudaGetSymbolAddress), so a context recreated after cudaDeviceReset is
 *   served too. All calls on a device share the one array and
 *   it keeps the last call's contents, which no call relies on; calls that can
 *   overlap on the GPU (different streams, or different host threads without
 *   ordering) race on it and must be serialized by the caller. A bounded wait
 *   that gave up inside the kernel is reported by ssd_fwd_no_alloc_check.
 */
SSD_API ssd_status_t ssd_fwd_no_alloc(const ssd_shape_t* shape,
                                      const void* x, const float* dt, const float* A,
                                      const void* B, const void* C, const float* D,
                                      const float* initial_states,
                                      void* y, float* final_states, void* stream);

/* Device-side status of the last ssd_fwd_no_alloc on the current device (same
 * shape): ssd_fwd_check on the static scratch array. Waits for `stream`. */
SSD_API ssd_status_t ssd_fwd_no_alloc_check(const ssd_shape_t* shape, void* stream);

/*
 * Device-side status of the last ssd_fwd that ran with `workspace` (same shape
 * and workspace as that call). Waits for `stream`, so call it after the outputs
 * are needed anyway. Returns SSD_OK, or SSD_ERR_TIMEOUT when a bounded wait
 * inside the fused kernel gave up (about 2 s: a chain hand-off or a hand-off
 * between the kernel's warp roles that never completed); that kernel then left
 * its outputs incomplete but the CUDA context usable, and ssd_last_error_detail()
 * names the wait. The step paths have no device-side waits and always report
 * SSD_OK. There is no counterpart in the pages; it exists because the fused
 * kernel's waits are bounded instead of hanging the GPU.
 */
SSD_API ssd_status_t ssd_fwd_check(const ssd_shape_t* shape, const void* workspace,
                                   size_t workspace_bytes, void* stream);

/* Bytes of device workspace ssd_fwd_host needs (inputs, outputs and ssd_fwd's
 * own workspace are staged there). */
SSD_API ssd_status_t ssd_fwd_host_workspace_size(const ssd_shape_t* shape, size_t* bytes);

/*
 * Same computation as ssd_fwd on HOST buffers: copies the inputs to the device
 * workspace, runs ssd_fwd there, copies y (and final_states when non-NULL)
 * back, and returns when everything is done, so the host outputs are ready on
 * return. The batch is processed in up to 8 slices of rows: the forward of a
 * slice runs on `stream` while two copy streams copy the next slice in and
 * the previous one out; the copies start after the work already queued on
 * `stream`. The copy streams and their events come from a per-device pool
 * that the library keeps until the process exits: the first call creates a
 * set, later calls reuse it (concurrent calls each take their own set), so a
 * steady stream of calls creates no CUDA objects. Host buffers should be page-locked for full
 * copy bandwidth; pageable memory works but is slower. The device workspace
 * must hold ssd_fwd_host_workspace_size() bytes. Returns SSD_ERR_TIMEOUT (as
 * ssd_fwd_check) when the fused kernel's bounded waits gave up.
 */
SSD_API ssd_status_t ssd_fwd_host(const ssd_shape_t* shape,
                          const void* x, const float* dt, const float* A,
                          const void* B, const void* C, const float* D,
                          const float* initial_states,
                          void* y, float* final_states,
                          void* device_workspace, size_t workspace_bytes, void* stream);

/*
 * Packed variable-length documents (Knowl 8, variable-length processing:
 * sequences of different lengths are concatenated into one flat sequence with
 * no padding, and the transition a_t is 0 at each document's first token, so
 * the state restarts at every boundary). Equivalent to one ssd_fwd per
 * document on its slice of the pack, computed in one pass over the pack.
 *   shape              batch = 1; seqlen = T, the packed length; the other
 *                      fields as for ssd_fwd (chunk_size not used). Supported:
 *                      dtype SSD_BF16, headdim 64, dstate a multiple of 16 up
 *                      to 256 (else SSD_ERR_UNSUPPORTED, nothing enqueued).
 *   x, dt, B, C, y     the pack, laid out as ssd_fwd's tensors with b = 1.
 *   A, D               as for ssd_fwd.
 *   cu_seqlens         DEVICE int32 [n_docs + 1]: document k is tokens
 *                      cu_seqlens[k] .. cu_seqlens[k+1] - 1; the list must
 *                      run from 0 to T, non-decreasing (empty documents are
 *                      allowed). It is read on the device: a malformed list is
 *                      clamped into [0, T] (nothing outside the pack is read or
 *                      written) and reported by ssd_fwd_varlen_check as
 *                      SSD_ERR_INVALID_ARG.
 *   n_docs             >= 0 (0 only with T = 0: nothing to do).
 *   initial_states     [n_docs, H, P, N] fp32 or NULL (zeros).
 *   final_states       [n_docs, H, P, N] fp32 or NULL (not written); an empty
 *                      document's final state is its initial state.
 *   workspace          ssd_fwd_varlen_workspace_size() bytes, 16-byte aligned;
 *                      holds the call's status words and the document order.
 * Two kernel launches: the documents are ranked by length (identity order
 * beyond 8192 documents) and checked, then the single-pass kernel runs one
 * unit per (document, head block), the longest documents first; a document's
 * tiles start at its first token, its tokens past the end get dt = 0 and rows
 * of the next document are never written.
 */
SSD_API ssd_status_t ssd_fwd_varlen_workspace_size(const ssd_shape_t* shape, int64_t n_docs,
                                                   size_t* bytes);
SSD_API ssd_status_t ssd_fwd_varlen(const ssd_shape_t* shape,
                                    const void* x, const float* dt, const float* A,
                                    const void* B, const void* C, const float* D,
                                    const int32_t* cu_seqlens, int64_t n_docs,
                                    const float* initial_states,
                                    void* y, float* final_states,
                                    void* workspace, size_t workspace_bytes, void* stream);
/* Status of the last ssd_fwd_varlen on `workspace` (waits for `stream`):
 * SSD_ERR_INVALID_ARG for a malformed cu_seqlens, SSD_ERR_TIMEOUT when a
 * bounded wait inside the kernel gave up, else SSD_OK. */
SSD_API ssd_status_t ssd_fwd_varlen_check(const ssd_shape_t* shape, int64_t n_docs,
                                          const void* workspace, size_t workspace_bytes,
                                          void* stream);

/*
 * The forward followed by the gate and normalisation of the Mamba-2 block
 * (Knowl 6, step 4):
 *     y   = ssd_fwd(x, dt, A, B, C, D, initial_states)
 *     out = ssd_gated_rmsnorm(y, z, norm_weight, group_size, eps)
 * with y rounded to dtype in between, as the two separate calls would have it.
 *   fuse = 1: when ssd_fwd_plan names the single-pass kernel and group_size
 *     divides a head's 64 channels (8, 16, 32 or 64), the kernel gates and
 *     normalises each staged row before storing it: out is written instead of
 *     y, so y needs neither memory nor a round trip through HBM. The gate's
 *     arithmetic then runs on the kernel's four store warps, which makes the
 *     forward slower than the two separate launches (measured at the 2.7B
 *     layer shape: 0.444 ms against 0.258 ms); it trades time for the y buffer.
 *   fuse = 0, or a shape / group size the kernel cannot gate: y is written to
 *     the workspace and the gate kernel follows (two launches more).
 *   z                  [b, T, H, P] in dtype (16-byte aligned), the gate branch.
 *   norm_weight        [H * P] fp32, 16-byte aligned.
 *   group_size, eps    as for ssd_gated_rmsnorm (group_size divides H * P).
 *   out                [b, T, H, P] in dtype, in y's place for every rule of ssd_fwd.
 *   final_states       as for ssd_fwd.
 *   workspace          ssd_fwd_gated_workspace_size() bytes (same group_size and
 *                      fuse): ssd_fwd's workspace, plus y when the gate is separate.
 * z, norm_weight must not overlap out, final_states or the workspace.
 */
SSD_API ssd_status_t ssd_fwd_gated_workspace_size(const ssd_shape_t* shape, int64_t group_size,
                                                  int fuse, size_t* bytes);
SSD_API ssd_status_t ssd_fwd_gated(const ssd_shape_t* shape,
                                   const void* x, const float* dt, const float* A,
                                   const void* B, const void* C, const float* D,
                                   const float* initial_states,
                                   const void* z, const float* norm_weight, int64_t group_size,
                                   float eps, int fuse, void* out, float* final_states,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * Recurrent (linear) form for the decoding mode of the layer (Knowl 1, linear
 * form: each new token costs O(P N) per head, however long the context): runs
 * shape->seqlen tokens per batch row from `state` and leaves the state after
 * the last one in `state`:
 *     a = exp(dt[b,t,h] * A[h])
 *     state[b,h,p,n] <- a * state[b,h,p,n] + dt[b,t,h] * x[b,t,h,p] * B[b,t,g,n]
 *     y[b,t,h,p] = sum_n C[b,t,g,n] * state[b,h,p,n] + D[h] * x[b,t,h,p]
 * i.e. ssd_fwd with initial_states = final_states = state, token by token.
 *   x, dt, A, B, C, D, y   as for ssd_fwd (seqlen = tokens of this call, usually 1;
 *                          seqlen 0 leaves state unchanged and writes no y).
 *   state                  [b,H,P,N] fp32, read and overwritten in place; must
 *                          not overlap any input or y.
 *   shape->chunk_size      not used (any value).
 * No workspace; one kernel launch (none when batch or seqlen is 0). The state
 * is read once and written once per call, so a call is an HBM stream of
 * 8 b H P N bytes plus the token's inputs; long prompts belong to ssd_fwd,
 * whose final_states then seed this call.
 */
SSD_API ssd_status_t ssd_step(const ssd_shape_t* shape,
                              const void* x, const float* dt, const float* A,
                              const void* B, const void* C, const float* D,
                              float* state, void* y, void* stream);

/*
 * Gate and normalisation that follow the layer in the Mamba-2 block (Knowl 6,
 * step 4: the layer output is gated by SiLU of the gate branch z, then
 * RMS-normalised before the output projection). Per token (b, t) and group of
 * group_size contiguous channels of its H*P channels (head-major, as y):
 *     v_c   = y_c * z_c / (1 + exp(-z_c))
 *     out_c = v_c / sqrt(mean over the group of v^2 + eps) * weight_c
 *   shape          batch, seqlen, nheads, headdim, dtype are used (the others
 *                  only have to be valid for ssd_fwd, chunk_size excepted).
 *   y, z, out      [b, T, H, P] in dtype (16-byte aligned); out must not overlap
 *                  y, z or weight.
 *   weight         [H * P] fp32.
 *   group_size     divides H * P (H * P for one group per token).
 *   eps            >= 0, finite (with eps = 0 a group whose gated values are
 *                  all 0 gives NaN, 0/0, as the formula does).
 * fp32 arithmetic (SiLU's exponential and division on the special-function
 * unit, a few ulp), out rounded once to dtype. One kernel launch.
 */
SSD_API ssd_status_t ssd_gated_rmsnorm(const ssd_shape_t* shape, const void* y, const void* z,
                                       const float* weight, int64_t group_size, float eps,
                                       void* out, void* stream);

/* ---- Sequence (context) parallelism (Knowl 8: the sequence is split along its
 * length across workers; each runs its slice and only the boundary state
 * travels). ----
 * Rank r of R holds the contiguous slice r of every batch row's sequence (any
 * lengths, zero allowed); all ranks share batch, nheads, headdim, ngroups,
 * dstate, chunk_size and dtype, seqlen being the rank's own slice length. Per
 * rank and call:
 *   1. ssd_cp_begin: the state the slice reaches, then this
 *      rank's record = [s (b H P N floats) | alpha (b H floats) | pad], where
 *      s is the state the slice reaches from a zero state (rank 0: from the
 *      sequence's initial_states) and alpha[b,h] = prod_{t in slice} a_t.
 *   2. the caller all-gathers the records of every rank, in rank order, into
 *      one buffer of R * record_floats floats (NCCL all-gather, or any
 *      collective with that result);
 *   3. ssd_cp_end: rank r's entering state h_in = fold over k < r of
 *      h <- alpha_k h + s_k from h = 0 (rank 0: initial_states), then the
 *      slice's forward from h_in: y of the slice and, in final_states, the
 *      state after the slice (on the last rank, the sequence's final state).
 * The result equals ssd_fwd over the whole sequence up to rounding. Where
 * ssd_fwd takes the single-pass kernel (bf16, head dim 64, state a multiple of
 * 16 up to 256), step 1 is the segment-state pass over the slice with its scan
 * (two launches) and step 3 is the fold plus ssd_fwd from h_in; otherwise both
 * run the four-step kernels (chunk cumsum and chunk states in step 1, state
 * passing and chunk scan in step 3). The exchange is one record per rank
 * (about 1 MiB at 32 heads x 64 x 128). */

/* Floats in one rank's record (b*H*P*N + b*H, rounded up to a multiple of 4). */
SSD_API ssd_status_t ssd_cp_record_floats(const ssd_shape_t* shape, size_t* floats);

/* Bytes of the device workspace ssd_cp_begin fills and ssd_cp_end reads. */
SSD_API ssd_status_t ssd_cp_workspace_size(const ssd_shape_t* shape, size_t* bytes);

/* Step 1 on this rank's slice. initial_states: the sequence's initial state on
 * rank 0, NULL on every other rank (and NULL on rank 0 for a zero state).
 * record: ssd_cp_record_floats() floats (16-byte aligned) receiving the record.
 * workspace: ssd_cp_workspace_size() bytes, kept untouched until ssd_cp_end
 * (it carries what step 3 needs from step 1: A, or the slice's chunk sums and
 * chunk states). */
SSD_API ssd_status_t ssd_cp_begin(const ssd_shape_t* shape,
                                  const void* x, const float* dt, const float* A,
                                  const void* B, const float* initial_states,
                                  float* record, void* workspace, size_t workspace_bytes,
                                  void* stream);

/* Step 3 on this rank's slice. records: the gathered records of all nranks
 * ranks (nranks * record_floats floats, rank k's at offset k * record_floats);
 * only those of ranks below `rank` are read. initial_states: as passed to
 * ssd_cp_begin on rank 0 (ignored on other ranks). y: the slice's output
 * [b, seqlen, H, P]. final_states (nullable): the state after the slice.
 * workspace: the one ssd_cp_begin filled for this slice. */
SSD_API ssd_status_t ssd_cp_end(const ssd_shape_t* shape, int nranks, int rank,
                                const float* records, const float* initial_states,
                                const void* x, const float* dt,
                                const void* B, const void* C, const float* D,
                                void* y, float* final_states,
                                void* workspace, size_t workspace_bytes, void* stream);

/* ---- The four steps of the block-decomposition algorithm, one call each. ----
 * ssd_fwd runs the same steps (or a fused equivalent); these entry points
 * expose each one with its intermediate tensors for callers that need them:
 *     cs       [b, H, nc, Q]      fp32, nc = ceil(T / Q)
 *     states   [b, nc, H, P, N]   fp32
 */

/* Step 1 (Knowl 2, "intra-chunk cumulative products of A", kept as log sums):
 * cs[b,h,c,k] = sum_{k'<=k} dt[b, cQ+k', h] * A[h], inclusive, within chunk c.
 * Entries past the end of a partial last chunk repeat its last value. */
SSD_API ssd_status_t ssd_chunk_cumsum(const ssd_shape_t* shape, const float* dt, const float* A,
                              float* cs, void* stream);

/* Step 2 (Knowl 2, "right factor chunk state" B^T (decayed X)):
 * states[b,c,h,p,n] = sum_{k in chunk c} exp(cs[..,last] - cs[..,k]) * dt_k * x_k[p] * B_k[n],
 * the state chunk c alone produces from a zero state. */
SSD_API ssd_status_t ssd_chunk_state(const ssd_shape_t* shape, const void* x, const float* dt,
                             const void* B, const float* cs, float* states, void* stream);

/* Step 3 (Knowl 2, inter-chunk recurrence h_{c+1} = (prod_t a_t) h_c + S_c):
 * entry_states[b,c] receives h_c, the state entering chunk c (h_0 = initial_states
 * or 0); final_states (nullable) receives h_nc. */
SSD_API ssd_status_t ssd_state_passing(const ssd_shape_t* shape, const float* states, const float* cs,
                               const float* initial_states, float* entry_states,
                               float* final_states, void* stream);

/* Step 4 (Knowl 2, Y_diag + Y_off per chunk, plus the D skip term):
 * y[j] = sum_{i<=j in chunk} (C_j . B_i) exp(cs_j - cs_i) dt_i x_i
 *        + exp(cs_j) C_j . h_c + D_h x_j. */
SSD_API ssd_status_t ssd_chunk_scan(const ssd_shape_t* shape, const void* x, const float* dt,
                            const void* B, const void* C, const float* D, const float* cs,
                            const float* entry_states, void* y, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H_ */
