// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {

struct Dims {
    int64_t b, T, H, P, G, N, Q, nc;
    int dtype;  // ssd_dtype_t
};

inline Dims make_dims(const ssd_shape_t& s) {
    Dims d;
    d.b = s.batch; d.T = s.seqlen; d.H = s.nheads; d.P = s.headdim; d.G = s.ngroups;
    d.N = s.dstate; d.Q = s.chunk_size; d.dtype = s.dtype;
    d.nc = d.T > 0 ? (d.T + d.Q - 1) / d.Q : 0;
    return d;
}

// CUDA-core kernels (any supported shape, fp32 or bf16 storage, fp32 math).
cudaError_t launch_chunk_cumsum(const Dims& d, const float* dt, const float* A, float* cs,
                                cudaStream_t st);
cudaError_t launch_chunk_state_simt(const Dims& d, const void* x, const float* dt, const void* B,
                                    const float* cs, float* states, cudaStream_t st);
cudaError_t launch_state_passing(const Dims& d, const float* states, const float* cs,
                                 const float* init, float* entry, float* final_states,
                                 cudaStream_t st);
cudaError_t launch_chunk_scan_simt(const Dims& d, const void* x, const float* dt, const void* B,
                                   const void* C, const float* D, const float* cs,
                                   const float* entry, void* y, cudaStream_t st);
// Tensor-core path (sm_100a tcgen05): bf16, head dim 64, state dim 128, chunk 128/256.
bool tc_supported(const Dims& d);
// cuTensorMapEncodeTiled is reachable through the runtime's driver entry points.
bool tma_available();
cudaError_t launch_chunk_state_tc(const Dims& d, const void* x, const float* dt, const void* B,
                                  const float* cs, float* states, cudaStream_t st);
cudaError_t launch_chunk_scan_tc(const Dims& d, const void* x, const float* dt, const void* B,
                                 const void* C, const float* D, const float* cs,
                                 const float* entry, void* y, cudaStream_t st);
int pick_kheads(int64_t heads_per_group);
// TMA maps of x, B, C (bf16, 4-D, 64 x 1 x 128 x 1 boxes) and y (64 x 1 x 32 x 1 boxes),
// 128-byte swizzle.
bool make_tc_maps(const Dims& d, const void* x, const void* B, const void* C, const void* y,
                  CUtensorMap* maps);

// Single-pass forward (ssd_fused.cu): bf16, head dim 64, state dim a multiple of 16
// up to 256. State capacity of the kernel variant for N (128 or 256; 0: unsupported).
int fused_state_capacity(int64_t N);
int fused_kheads(int64_t H, int64_t G, int ns);
// ints of the kernel's sync area: ticket, error word, one flag per (b, segment, head)
size_t fused_sync_ints(const Dims& d, int nseg);
struct FusedLaunch {
    Dims d;
    const CUtensorMap* maps;   // x, B, C, y
    const float* dt;
    const float* A;
    const float* D;
    const float* init;         // [b,H,P,N] or null
    float* finalbuf;           // [b,H,P,N] final states, or null
    float* segbuf;             // [b,nslot,H,P,N] states entering segments 1.. (nseg > 1)
    int* sync_ints;            // fused_sync_ints ints, zeroed by the caller
    int kheads, seg_tiles, nseg;
    int seg_first;             // tiles of segment 0 (chained only; 0: seg_tiles)
    int chained;               // segment s > 0 takes its entering state from segment s - 1's unit
    int nslot;                 // segbuf slots per batch row; 0: nseg
    int stall;                 // test builds: make chain waits run out
    void* y;                   // [b,T,H,P] bf16 (the map's tensor): rows of partial tiles
    // gate and norm after the layer, fused into the stores (z null: y stored as is):
    // out = RMSNorm over groups of gs channels of y * SiLU(z), times nw; y is then the
    // output buffer and the map is over it. gs divides 64 and is a multiple of 8.
    const void* z;
    const float* nw;
    int gs;
    float eps;
    // packed documents (d.b == 1, nseg == 1): document k is tokens cu[k] .. cu[k+1]-1;
    // init / finalbuf are [ndoc,H,P,N]; units run in `order` (varlen_order output)
    const int* cu;
    const int* order;
    int ndoc;
};
cudaError_t launch_fused(const FusedLaunch& a, cudaStream_t st);

// Whether the single-pass kernel's stores can apply the gate and norm for this
// group size (groups inside one head's 64 channels).
inline bool fused_gate_ok(int64_t group_size) {
    return group_size >= 8 && group_size <= 64 && 64 % group_size == 0 && group_size % 8 == 0;
}

// Packed documents: order[ndoc] = documents by decreasing length (ties by index;
// identity order above varlen_sort_max() documents), and *bad = 1 when cu is not a
// non-decreasing list from 0 to T.
int varlen_sort_max();
cudaError_t launch_varlen_order(const int* cu, int ndoc, int64_t T, int* order, int* bad,
                                cudaStream_t st);

// Segment states (ssd_segment.cu): for each segment s < nseg_out of seg_tiles tiles,
// the state it reaches from zero, written to segbuf slot s + 1 ([b,nslot,H,P,N]), and
// its decay 2^(sum dt A log2 e) to decay[b,nseg,H] at s. The scan over segments then
// turns slot s (1 <= s <= nseg_out) into the state entering segment s (init entering
// segment 0) and, when `final_out` is given, writes the state after segment
// nseg_out - 1 there (and with `alpha_out` [b,H] the decay over segments
// 0 .. nseg_out - 1); with store = false the slots are left as they are (only
// final_out and alpha_out are written). Bounded waits that give up set *error.
int segment_max_tiles();
cudaError_t launch_segment_states(const Dims& d, const CUtensorMap* maps, const float* dt,
                                  const float* A, float* segbuf, float* decay, int* error,
                                  int seg_tiles, int nseg, int nslot, int nseg_out, int kheads,
                                  cudaStream_t st);
cudaError_t launch_segment_scan(const Dims& d, const float* init, float* segbuf, const float* decay,
                                int nseg, int nslot, int nseg_out, float* final_out,
                                cudaStream_t st, float* alpha_out = nullptr, bool store = true);

// Recurrent form for a few tokens per sequence, state [b,H,P,N] updated in place.
struct StepLayout {
    int W;             // state elements per load (4 when N % 4 == 0, else 1)
    int L;             // lanes sharing one state row
    int K;             // W-wide pieces of a row per lane
    int rows_per_cta;  // state rows one CTA owns
};
StepLayout step_layout(int64_t N);
cudaError_t launch_step(const Dims& d, const void* x, const float* dt, const float* A, const void* B,
                        const void* C, const float* D, float* state, void* y, cudaStream_t st);

// Sequence parallelism: alpha[b,h] = prod of a_t over the slice (from cs), and the fold
// of ranks 0..rank-1's records [state b*H*P*N | alpha b*H] into rank's entering state.
cudaError_t launch_slice_decay(const Dims& d, const float* cs, float* alpha, cudaStream_t st);
cudaError_t launch_cp_fold(const Dims& d, const float* records, int64_t rec_floats, int rank,
                           float* h_in, cudaStream_t st);

// Gate and RMSNorm after the layer: out = (y * SiLU(z)) / rms over groups of group_size
// channels * weight, for b*T rows of H*P channels.
cudaError_t launch_gated_rmsnorm(const Dims& d, const void* y, const void* z, const float* w,
                                 int64_t group_size, float eps, void* out, cudaStream_t st);

// Sets the message ssd_last_error_detail() returns on the calling host thread.
void set_error_detail(const char* msg);

cudaError_t launch_copy_or_zero_states(const Dims& d, const float* init, float* final_states,
                                       cudaStream_t st);

}  // namespace ssd
