// Sequence (context) parallelism: the two small kernels around the one exchange
// step ("Transformers are SSMs: Generalized Models and Efficient Algorithms
// Through Structured State Space Duality", Knowl 8, sequence / context
// parallelism: each worker runs its slice of the sequence and only the boundary
// state is passed on).
//
// A rank's slice acts on the state entering it as the affine map
//     h -> alpha * h + s,   alpha[b,h] = prod_{t in slice} a_t,
// s being the state the slice reaches from a zero state (or, on rank 0, from
// the sequence's initial state). Composing these maps over ranks 0..r-1 gives
// rank r's entering state; that fold is a linear recurrence over ranks, the
// same one as the state passing between chunks (Knowl 2), one level up.
#include <cuda_runtime.h>

#include "ssd_internal.h"

namespace ssd {
namespace {

// alpha[b,h] = exp(sum over the slice's chunks of the chunk's total log decay),
// the last valid entry of each chunk's inclusive cumulative sum of dt*A.
__global__ void slice_decay_kernel(const float* __restrict__ cs, float* __restrict__ alpha,
                                   int64_t BH, int64_t T, int Q, int64_t nc) {
    const int64_t bh = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (bh >= BH) return;
    float sum = 0.f;
    for (int64_t c = 0; c < nc; ++c) {
        const int len = (int)min((int64_t)Q, T - c * Q);
        sum += cs[(bh * nc + c) * Q + len - 1];
    }
    alpha[bh] = expf(sum);
}

// h_in[i] for rank `rank`: h = 0, then h = alpha_k * h + s_k for k = 0 .. rank-1,
// record k at records + k * rec_floats = [s_k (b H P N floats) | alpha_k (b H)].
__global__ void cp_fold_kernel(const float* __restrict__ records, int64_t rec_floats, int rank,
                               int64_t n_state, int64_t PN, float* __restrict__ h_in) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_state) return;
    const int64_t bh = i / PN;
    float h = 0.f;
    for (int k = 0; k < rank; ++k) {
        const float* rec = records + (int64_t)k * rec_floats;
        h = fmaf(rec[n_state + bh], h, rec[i]);
    }
    h_in[i] = h;
}

}  // namespace

cudaError_t launch_slice_decay(const Dims& d, const float* cs, float* alpha, cudaStream_t st) {
    const int64_t BH = d.b * d.H;
    if (BH == 0) return cudaSuccess;
    slice_decay_kernel<<<(unsigned)((BH + 255) / 256), 256, 0, st>>>(cs, alpha, BH, d.T, (int)d.Q, d.nc);
    return cudaGetLastError();
}

cudaError_t launch_cp_fold(const Dims& d, const float* records, int64_t rec_floats, int rank,
                           float* h_in, cudaStream_t st) {
    const int64_t n = d.b * d.H * d.P * d.N;
    if (n == 0) return cudaSuccess;
    cp_fold_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(records, rec_floats, rank, n,
                                                                d.P * d.N, h_in);
    return cudaGetLastError();
}

}  // namespace ssd
