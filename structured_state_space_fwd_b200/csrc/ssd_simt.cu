// CUDA-core (FFMA) kernels for the four steps of the block-decomposition SSD
// algorithm ("Transformers are SSMs", Knowl 2). They serve every supported
// shape and both storage types (fp32, bf16; math in fp32), and are the whole
// path for fp32 inputs, where tensor-core rounding would exceed a 1e-5 budget.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ssd_internal.h"

namespace ssd {
namespace {

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void from_f(float* p, float v) { *p = v; }
__device__ __forceinline__ void from_f(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// ---------------------------------------------------------------------------
// Step 1: cs[b,h,c,k] = inclusive cumsum over k of dt*A within chunk c.
// Block = (chunk c, 32-head tile, batch b), 256 threads. The [Q x 32] tile of
// dt is read row by row (32 consecutive heads per token, coalesced), scaled by
// A, then each warp scans 4 heads: a lane owns ceil(Q/32) consecutive tokens,
// sums them sequentially and the lane totals are combined by a shuffle scan.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) chunk_cumsum_kernel(const float* __restrict__ dt,
                                                           const float* __restrict__ A,
                                                           float* __restrict__ cs, int64_t T,
                                                           int64_t H, int Q, int64_t nc) {
    extern __shared__ float tile[];  // [Q][33]
    const int c = blockIdx.x;
    const int64_t h0 = (int64_t)blockIdx.y * 32;
    const int64_t b = blockIdx.z;
    const int tid = threadIdx.x;
    for (int idx = tid; idx < Q * 32; idx += 256) {
        const int k = idx >> 5, hh = idx & 31;
        const int64_t t = (int64_t)c * Q + k;
        const int64_t h = h0 + hh;
        float v = 0.f;
        if (t < T && h < H) v = dt[(b * T + t) * H + h] * A[h];
        tile[k * 33 + hh] = v;
    }
    __syncthreads();
    const int warp = tid >> 5, lane = tid & 31;
    const int per = (Q + 31) / 32;
    for (int hh = warp; hh < 32; hh += 8) {
        const int64_t h = h0 + hh;
        if (h >= H) break;
        const int kbeg = lane * per;
        const int kend = min(Q, kbeg + per);
        float run = 0.f;
        for (int k = kbeg; k < kend; ++k) run += tile[k * 33 + hh];
        // exclusive scan of the lane totals
        float incl = run;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        float acc = incl - run;
        float* out = cs + ((b * H + h) * nc + c) * Q;
        for (int k = kbeg; k < kend; ++k) {
            acc += tile[k * 33 + hh];
            out[k] = acc;
        }
    }
}

// ---------------------------------------------------------------------------
// Step 2: states[b,c,h,p,n] = sum_k w_k x_k[p] B_k[n], w_k = exp(cs_last - cs_k) dt_k.
// Block = (32x32 tile of (p, n), (c, h), b); thread (ty, tx) accumulates rows
// p = 4*ty .. 4*ty+3 of column n = tx over 32-token tiles staged in shared memory.
// ---------------------------------------------------------------------------
template <typename Tin, bool kAccurateExp>
__global__ void __launch_bounds__(256) chunk_state_simt_kernel(
    const Tin* __restrict__ x, const float* __restrict__ dt, const Tin* __restrict__ Bm,
    const float* __restrict__ cs, float* __restrict__ states, int64_t T, int64_t H, int64_t P,
    int64_t G, int64_t N, int Q, int64_t nc) {
    __shared__ float xs[32][33];
    __shared__ float bs[32][33];
    const int64_t ntn = (N + 31) / 32;
    const int64_t p0 = (blockIdx.x / ntn) * 32, n0 = (blockIdx.x % ntn) * 32;
    const int64_t c = blockIdx.y / H, h = blockIdx.y % H;
    const int64_t b = blockIdx.z;
    const int64_t g = h / (H / G);
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int64_t t0 = c * Q;
    const int len = (int)min((int64_t)Q, T - t0);
    const float* csc = cs + ((b * H + h) * nc + c) * Q;
    const float cs_last = csc[len - 1];
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k0 = 0; k0 < len; k0 += 32) {
        for (int idx = threadIdx.x; idx < 32 * 32; idx += 256) {
            const int kk = idx >> 5, j = idx & 31;
            const int k = k0 + kk;
            float xv = 0.f, bv = 0.f;
            if (k < len) {
                const int64_t t = t0 + k;
                const float arg = cs_last - csc[k];
                const float w = (kAccurateExp ? expf(arg) : __expf(arg)) * dt[(b * T + t) * H + h];
                if (p0 + j < P) xv = w * to_f(x[((b * T + t) * H + h) * P + p0 + j]);
                if (n0 + j < N) bv = to_f(Bm[((b * T + t) * G + g) * N + n0 + j]);
            }
            xs[kk][j] = xv;
            bs[kk][j] = bv;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) {
            const float bv = bs[kk][tx];
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[r] = fmaf(xs[kk][ty * 4 + r], bv, acc[r]);
        }
        __syncthreads();
    }
    float* out = states + ((b * nc + c) * H + h) * P * N;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int64_t p = p0 + ty * 4 + r, n = n0 + tx;
        if (p < P && n < N) out[p * N + n] = acc[r];
    }
}

// ---------------------------------------------------------------------------
// Step 3: sequential over chunks, elementwise over (p, n):
//   entry[b,c,h] = h_c;  h_{c+1} = exp(cs[b,h,c,last]) h_c + S[b,c,h].
// One thread per state element; consecutive threads take consecutive (p, n),
// so every load and store is coalesced.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) state_passing_kernel(
    const float* __restrict__ S, const float* __restrict__ cs, const float* __restrict__ init,
    float* __restrict__ entry, float* __restrict__ final_states, int64_t T, int64_t H,
    int64_t PN, int Q, int64_t nc) {
    const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;
    const int64_t h = blockIdx.y, b = blockIdx.z;
    if (e >= PN) return;
    float hv = init ? init[(b * H + h) * PN + e] : 0.f;
    for (int64_t c = 0; c < nc; ++c) {
        const int len = (int)min((int64_t)Q, T - c * Q);
        if (entry) entry[((b * nc + c) * H + h) * PN + e] = hv;
        const float decay = expf(cs[((b * H + h) * nc + c) * Q + len - 1]);
        hv = fmaf(decay, hv, S[((b * nc + c) * H + h) * PN + e]);
    }
    if (final_states) final_states[(b * H + h) * PN + e] = hv;
}

// T == 0: final = initial (or 0).
__global__ void copy_or_zero_kernel(const float* __restrict__ init, float* __restrict__ out,
                                    int64_t n) {
    const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (i < n) out[i] = init ? init[i] : 0.f;
}

// ---------------------------------------------------------------------------
// Step 4: y[j] = sum_{i<=j} (C_j . B_i) exp(cs_j - cs_i) dt_i x_i
//              + exp(cs_j) sum_n C_j[n] h_c[p][n] + D_h x_j[p]
// Block = (32-row tile jt of the chunk, (c, h), b), 256 threads: thread (r, q)
// owns row j = 32*jt + r and columns p = q + 8m. Causal: only column tiles
// it <= jt are visited and entries with i > j are zeroed before the exponential.
// ---------------------------------------------------------------------------
template <typename Tin, bool kAccurateExp>
__global__ void __launch_bounds__(256) chunk_scan_simt_kernel(
    const Tin* __restrict__ x, const float* __restrict__ dt, const Tin* __restrict__ Bm,
    const Tin* __restrict__ Cm, const float* __restrict__ D, const float* __restrict__ cs,
    const float* __restrict__ entry, Tin* __restrict__ y, int64_t T, int64_t H, int64_t P,
    int64_t G, int64_t N, int Q, int64_t nc) {
    extern __shared__ float sm[];
    const int NS = (int)N + 1;            // padded row stride of C / B tiles
    const int PS = (int)P + 1;            // padded row stride of the x tile
    float* Cs = sm;                       // [32][NS]
    float* Bs = Cs + 32 * NS;             // [32][NS]
    float* Xs = Bs + 32 * NS;             // [32][PS]
    float* Hs = Xs + 32 * PS;             // [P][33]
    float* Ms = Hs + P * 33;              // [32][33]
    float* csi = Ms + 32 * 33;            // [32]
    float* dti = csi + 32;                // [32]

    const int jt = blockIdx.x;
    const int64_t c = blockIdx.y / H, h = blockIdx.y % H;
    const int64_t b = blockIdx.z;
    const int64_t g = h / (H / G);
    const int64_t t0 = c * Q;
    const int len = (int)min((int64_t)Q, T - t0);
    const int j0 = jt * 32;
    if (j0 >= len) return;
    const int tid = threadIdx.x;
    const int r = tid >> 3, q = tid & 7;
    const int j = j0 + r;
    const bool jvalid = j < len;
    const float* csc = cs + ((b * H + h) * nc + c) * Q;
    const float csj = csc[min(j, len - 1)];
    const int mp = (int)((P + 7) / 8);

    // C rows of this tile
    for (int idx = tid; idx < 32 * N; idx += 256) {
        const int rr = idx / (int)N, n = idx % (int)N;
        const int jj = j0 + rr;
        Cs[rr * NS + n] = jj < len ? to_f(Cm[((b * T + t0 + jj) * G + g) * N + n]) : 0.f;
    }

    float acc[32], acc2[32];
#pragma unroll
    for (int m = 0; m < 32; ++m) { acc[m] = 0.f; acc2[m] = 0.f; }

    for (int i0 = 0; i0 <= j0; i0 += 32) {
        __syncthreads();
        for (int idx = tid; idx < 32 * N; idx += 256) {
            const int ii = idx / (int)N, n = idx % (int)N;
            const int i = i0 + ii;
            Bs[ii * NS + n] = i < len ? to_f(Bm[((b * T + t0 + i) * G + g) * N + n]) : 0.f;
        }
        for (int idx = tid; idx < 32 * P; idx += 256) {
            const int ii = idx / (int)P, p = idx % (int)P;
            const int i = i0 + ii;
            Xs[ii * PS + p] = i < len ? to_f(x[((b * T + t0 + i) * H + h) * P + p]) : 0.f;
        }
        if (tid < 32) {
            const int i = i0 + tid;
            csi[tid] = i < len ? csc[i] : 0.f;
            dti[tid] = i < len ? dt[(b * T + t0 + i) * H + h] : 0.f;
        }
        __syncthreads();
        // masked scores for row r, columns ii = q + 8s
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int ii = q + 8 * s;
            const int i = i0 + ii;
            float sc = 0.f;
            if (jvalid && i <= j && i < len) {
                float dot = 0.f;
                for (int n = 0; n < N; ++n) dot = fmaf(Cs[r * NS + n], Bs[ii * NS + n], dot);
                const float arg = csj - csi[ii];
                const float dec = kAccurateExp ? expf(arg) : __expf(arg);
                sc = dot * dec * dti[ii];
            }
            Ms[r * 33 + ii] = sc;
        }
        __syncthreads();
        for (int ii = 0; ii < 32; ++ii) {
            const float mv = Ms[r * 33 + ii];
#pragma unroll
            for (int m = 0; m < 32; ++m)
                if (m < mp && q + 8 * m < P) acc[m] = fmaf(mv, Xs[ii * PS + q + 8 * m], acc[m]);
        }
    }

    // contribution of the state entering the chunk: sum_n C_j[n] h_c[p][n]
    const float* hc = entry + ((b * nc + c) * H + h) * P * N;
    for (int n0 = 0; n0 < N; n0 += 32) {
        __syncthreads();
        for (int idx = tid; idx < P * 32; idx += 256) {
            const int p = idx >> 5, nn = idx & 31;
            Hs[p * 33 + nn] = (n0 + nn < N) ? hc[(int64_t)p * N + n0 + nn] : 0.f;
        }
        __syncthreads();
        const int nlim = (int)min((int64_t)32, N - n0);
        for (int nn = 0; nn < nlim; ++nn) {
            const float cv = Cs[r * NS + n0 + nn];
#pragma unroll
            for (int m = 0; m < 32; ++m)
                if (m < mp && q + 8 * m < P) acc2[m] = fmaf(cv, Hs[(q + 8 * m) * 33 + nn], acc2[m]);
        }
    }

    if (!jvalid) return;
    const float ej = kAccurateExp ? expf(csj) : __expf(csj);
    const float Dh = D ? D[h] : 0.f;
    const int64_t row = ((b * T + t0 + j) * H + h) * P;
#pragma unroll
    for (int m = 0; m < 32; ++m) {
        const int p = q + 8 * m;
        if (m < mp && p < P) {
            const float xv = to_f(x[row + p]);
            from_f(&y[row + p], acc[m] + ej * acc2[m] + Dh * xv);
        }
    }
}

inline size_t chunk_scan_smem(const Dims& d) {
    return sizeof(float) * (size_t)(2 * 32 * (d.N + 1) + 32 * (d.P + 1) + d.P * 33 + 32 * 33 + 64);
}

}  // namespace

cudaError_t launch_chunk_cumsum(const Dims& d, const float* dt, const float* A, float* cs,
                                cudaStream_t st) {
    if (d.b == 0 || d.nc == 0) return cudaSuccess;
    dim3 grid((unsigned)d.nc, (unsigned)((d.H + 31) / 32), (unsigned)d.b);
    size_t smem = sizeof(float) * (size_t)d.Q * 33;
    cudaError_t e = cudaFuncSetAttribute(chunk_cumsum_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    chunk_cumsum_kernel<<<grid, 256, smem, st>>>(dt, A, cs, d.T, d.H, (int)d.Q, d.nc);
    return cudaGetLastError();
}

cudaError_t launch_chunk_state_simt(const Dims& d, const void* x, const float* dt, const void* B,
                                    const float* cs, float* states, cudaStream_t st) {
    if (d.b == 0 || d.nc == 0) return cudaSuccess;
    dim3 grid((unsigned)(((d.P + 31) / 32) * ((d.N + 31) / 32)), (unsigned)(d.nc * d.H),
              (unsigned)d.b);
    if (d.dtype == SSD_BF16)
        chunk_state_simt_kernel<__nv_bfloat16, false><<<grid, 256, 0, st>>>(
            (const __nv_bfloat16*)x, dt, (const __nv_bfloat16*)B, cs, states, d.T, d.H, d.P, d.G,
            d.N, (int)d.Q, d.nc);
    else
        chunk_state_simt_kernel<float, true><<<grid, 256, 0, st>>>((const float*)x, dt,
                                                             (const float*)B, cs, states, d.T,
                                                             d.H, d.P, d.G, d.N, (int)d.Q, d.nc);
    return cudaGetLastError();
}

cudaError_t launch_state_passing(const Dims& d, const float* states, const float* cs,
                                 const float* init, float* entry, float* final_states,
                                 cudaStream_t st) {
    if (d.b == 0) return cudaSuccess;
    const int64_t PN = d.P * d.N;
    dim3 grid((unsigned)((PN + 255) / 256), (unsigned)d.H, (unsigned)d.b);
    state_passing_kernel<<<grid, 256, 0, st>>>(states, cs, init, entry, final_states, d.T, d.H,
                                                PN, (int)d.Q, d.nc);
    return cudaGetLastError();
}

cudaError_t launch_copy_or_zero_states(const Dims& d, const float* init, float* final_states,
                                       cudaStream_t st) {
    const int64_t n = d.b * d.H * d.P * d.N;
    if (n == 0 || !final_states) return cudaSuccess;
    copy_or_zero_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(init, final_states, n);
    return cudaGetLastError();
}

cudaError_t launch_chunk_scan_simt(const Dims& d, const void* x, const float* dt, const void* B,
                                   const void* C, const float* D, const float* cs,
                                   const float* entry, void* y, cudaStream_t st) {
    if (d.b == 0 || d.nc == 0) return cudaSuccess;
    dim3 grid((unsigned)((d.Q + 31) / 32), (unsigned)(d.nc * d.H), (unsigned)d.b);
    const size_t smem = chunk_scan_smem(d);
    cudaError_t e;
    if (d.dtype == SSD_BF16) {
        auto k = chunk_scan_simt_kernel<__nv_bfloat16, false>;
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k<<<grid, 256, smem, st>>>((const __nv_bfloat16*)x, dt, (const __nv_bfloat16*)B,
                                   (const __nv_bfloat16*)C, D, cs, entry, (__nv_bfloat16*)y, d.T,
                                   d.H, d.P, d.G, d.N, (int)d.Q, d.nc);
    } else {
        auto k = chunk_scan_simt_kernel<float, true>;
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k<<<grid, 256, smem, st>>>((const float*)x, dt, (const float*)B, (const float*)C, D, cs,
                                   entry, (float*)y, d.T, d.H, d.P, d.G, d.N, (int)d.Q, d.nc);
    }
    return cudaGetLastError();
}

}  // namespace ssd
