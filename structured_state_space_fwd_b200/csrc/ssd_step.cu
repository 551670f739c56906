// Recurrent (linear) form of the SSD layer, token by token from a state kept
// in HBM: the decoding mode of the layer ("Transformers are SSMs: Generalized
// Models and Efficient Algorithms Through Structured State Space Duality",
// Knowl 1, linear form). Per batch row b, head h (group g) and token t:
//
//     a      = exp(dt[b,t,h] * A[h])
//     h[p,n] = a * h[p,n] + dt[b,t,h] * x[b,t,h,p] * B[b,t,g,n]
//     y[b,t,h,p] = sum_n C[b,t,g,n] * h[p,n] + D[h] * x[b,t,h,p]
//
// Each row p of the state evolves on its own (it sees only x[p]), so a CTA
// owns a block of rows of one (b, h) and keeps them in registers for all the
// call's tokens: the state is read once and written once per call, whatever
// the token count. One token per call is an HBM stream of the state
// (8 P N bytes per head); that stream is what bounds the kernel.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ssd_internal.h"

namespace ssd {
namespace {

constexpr int kStepWarps = 4;
constexpr int kStepChunks = 4;   // W-wide pieces of state a thread holds

struct StepParams {
    const void* x;
    const float* dt;
    const float* A;
    const void* B;
    const void* C;
    const float* D;
    float* state;
    void* y;
    int64_t T, H, P, G, N;
    int L;     // lanes sharing one state row (power of two, <= 32)
};

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void store_out(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_out(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// W consecutive elements as fp32 (W = 4: one 16-byte (fp32) or 8-byte (bf16) load)
template <int W>
__device__ __forceinline__ void load_w(const float* p, float (&v)[W]) {
    if constexpr (W == 4) {
        const float4 q = *reinterpret_cast<const float4*>(p);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
#pragma unroll
        for (int w = 0; w < W; ++w) v[w] = p[w];
    }
}
template <int W>
__device__ __forceinline__ void load_w(const __nv_bfloat16* p, float (&v)[W]) {
    if constexpr (W == 4) {
        const uint2 q = *reinterpret_cast<const uint2*>(p);
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&q.y));
        v[0] = lo.x; v[1] = lo.y; v[2] = hi.x; v[3] = hi.y;
    } else {
#pragma unroll
        for (int w = 0; w < W; ++w) v[w] = __bfloat162float(p[w]);
    }
}
template <int W>
__device__ __forceinline__ void load_state(const float* p, float (&v)[W]) {
    if constexpr (W == 4) {
        const float4 q = __ldcs(reinterpret_cast<const float4*>(p));
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
#pragma unroll
        for (int w = 0; w < W; ++w) v[w] = __ldcs(p + w);
    }
}
template <int W>
__device__ __forceinline__ void store_state(float* p, const float (&v)[W]) {
    if constexpr (W == 4) {
        __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
    } else {
#pragma unroll
        for (int w = 0; w < W; ++w) __stcs(p + w, v[w]);
    }
}

// Thread layout: a warp covers 32 / L rows at a time, L lanes per row; lane j of
// a row holds the W-wide pieces n0 = (j + k L) W, k < K, of RS rows spaced
// kStepWarps * 32 / L apart. Grid (row blocks, H, batch). With 16-byte pieces
// the update runs on packed fp32x2 instructions and registers are capped so
// that 7 CTAs fit on an SM: many small CTAs keep more of the DRAM stream busy
// than few large ones.
template <typename E, int W, int K>
__global__ void __launch_bounds__(kStepWarps * 32, W == 4 ? 7 : 1) ssd_step_kernel(const StepParams prm) {
    constexpr int RS = kStepChunks / K > 0 ? kStepChunks / K : 1;
    const int L = prm.L;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int j = lane & (L - 1);
    const int rows_per_pass = kStepWarps * (32 / L);
    const int64_t h = blockIdx.y, b = blockIdx.z;
    const int64_t g = h / (prm.H / prm.G);
    const int64_t P = prm.P, N = prm.N, T = prm.T;
    const int64_t p_base = (int64_t)blockIdx.x * rows_per_pass * RS + warp * (32 / L) + (lane / L);
    const E* x = static_cast<const E*>(prm.x);
    const E* Bm = static_cast<const E*>(prm.B);
    const E* Cm = static_cast<const E*>(prm.C);
    E* y = static_cast<E*>(prm.y);
    const float Ah = prm.A[h];
    const float Dh = prm.D ? prm.D[h] : 0.f;

    bool row_ok[RS];
    bool piece_ok[K];
#pragma unroll
    for (int r = 0; r < RS; ++r) row_ok[r] = p_base + (int64_t)r * rows_per_pass < P;
#pragma unroll
    for (int k = 0; k < K; ++k) piece_ok[k] = (int64_t)(j + k * L) * W < N;

    float* st = prm.state + (b * prm.H + h) * P * N;
    float hs[RS][K][W];
#pragma unroll
    for (int r = 0; r < RS; ++r)
#pragma unroll
        for (int k = 0; k < K; ++k) {
            if (row_ok[r] && piece_ok[k])
                load_state<W>(st + (p_base + (int64_t)r * rows_per_pass) * N + (int64_t)(j + k * L) * W, hs[r][k]);
            else
#pragma unroll
                for (int w = 0; w < W; ++w) hs[r][k][w] = 0.f;
        }

    for (int64_t t = 0; t < T; ++t) {
        const int64_t bt = b * T + t;
        const float dtv = prm.dt[bt * prm.H + h];
        const float a = expf(dtv * Ah);
        float Bv[K][W], Cv[K][W];
        const int64_t bc = (bt * prm.G + g) * N;
#pragma unroll
        for (int k = 0; k < K; ++k) {
            if (piece_ok[k]) {
                load_w<W>(Bm + bc + (int64_t)(j + k * L) * W, Bv[k]);
                load_w<W>(Cm + bc + (int64_t)(j + k * L) * W, Cv[k]);
            } else {
#pragma unroll
                for (int w = 0; w < W; ++w) Bv[k][w] = Cv[k][w] = 0.f;
            }
        }
        const E* xt = x + (bt * prm.H + h) * P;
        E* yt = y + (bt * prm.H + h) * P;
#pragma unroll
        for (int r = 0; r < RS; ++r) {
            const int64_t p = p_base + (int64_t)r * rows_per_pass;
            const float xv = row_ok[r] ? to_f32(xt[p]) : 0.f;
            const float u = dtv * xv;
            float acc = 0.f;
            if constexpr (W == 4) {
                // packed fp32x2: two state elements per instruction
                const float2 a2 = make_float2(a, a), u2 = make_float2(u, u);
                float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
                for (int k = 0; k < K; ++k)
#pragma unroll
                    for (int w = 0; w < W; w += 2) {
                        float2 h2 = make_float2(hs[r][k][w], hs[r][k][w + 1]);
                        h2 = __ffma2_rn(a2, h2, __fmul2_rn(u2, make_float2(Bv[k][w], Bv[k][w + 1])));
                        acc2 = __ffma2_rn(make_float2(Cv[k][w], Cv[k][w + 1]), h2, acc2);
                        hs[r][k][w] = h2.x;
                        hs[r][k][w + 1] = h2.y;
                    }
                acc = acc2.x + acc2.y;
            } else {
#pragma unroll
                for (int k = 0; k < K; ++k)
#pragma unroll
                    for (int w = 0; w < W; ++w) {
                        hs[r][k][w] = fmaf(a, hs[r][k][w], u * Bv[k][w]);
                        acc = fmaf(Cv[k][w], hs[r][k][w], acc);
                    }
            }
            // sum over the L lanes of the row (aligned groups of L lanes)
            for (int off = L >> 1; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            if (j == 0 && row_ok[r]) store_out(yt + p, fmaf(Dh, xv, acc));
        }
    }

#pragma unroll
    for (int r = 0; r < RS; ++r)
#pragma unroll
        for (int k = 0; k < K; ++k)
            if (row_ok[r] && piece_ok[k])
                store_state<W>(st + (p_base + (int64_t)r * rows_per_pass) * N + (int64_t)(j + k * L) * W, hs[r][k]);
}

template <typename E, int W, int K>
cudaError_t launch_step_k(const StepParams& prm, int64_t b, cudaStream_t s) {
    constexpr int RS = kStepChunks / K > 0 ? kStepChunks / K : 1;
    const int64_t rows_per_cta = (int64_t)kStepWarps * (32 / prm.L) * RS;
    const dim3 grid((unsigned)((prm.P + rows_per_cta - 1) / rows_per_cta), (unsigned)prm.H, (unsigned)b);
    ssd_step_kernel<E, W, K><<<grid, kStepWarps * 32, 0, s>>>(prm);
    return cudaGetLastError();
}

template <typename E, int W>
cudaError_t launch_step_w(const StepParams& prm, int K, int64_t b, cudaStream_t s) {
    if constexpr (W == 4) {
        return K == 1 ? launch_step_k<E, 4, 1>(prm, b, s) : launch_step_k<E, 4, 2>(prm, b, s);
    } else {
        switch (K) {
            case 1: return launch_step_k<E, 1, 1>(prm, b, s);
            case 2: return launch_step_k<E, 1, 2>(prm, b, s);
            case 3: return launch_step_k<E, 1, 3>(prm, b, s);
            case 4: return launch_step_k<E, 1, 4>(prm, b, s);
            case 5: return launch_step_k<E, 1, 5>(prm, b, s);
            case 6: return launch_step_k<E, 1, 6>(prm, b, s);
            case 7: return launch_step_k<E, 1, 7>(prm, b, s);
            default: return launch_step_k<E, 1, 8>(prm, b, s);
        }
    }
}

}  // namespace

StepLayout step_layout(int64_t N) {
    StepLayout l;
    l.W = (N % 4 == 0) ? 4 : 1;
    const int64_t pieces = N / l.W;            // W-wide pieces per state row
    int L = 1;
    while (L < 32 && L < pieces) L <<= 1;
    l.L = L;
    l.K = (int)((pieces + L - 1) / L);          // <= 2 for W = 4, <= 8 for W = 1 (N <= 256)
    const int rs = kStepChunks / l.K > 0 ? kStepChunks / l.K : 1;
    l.rows_per_cta = kStepWarps * (32 / L) * rs;
    return l;
}

cudaError_t launch_step(const Dims& d, const void* x, const float* dt, const float* A, const void* B,
                        const void* C, const float* D, float* state, void* y, cudaStream_t s) {
    if (d.b == 0 || d.T == 0) return cudaSuccess;
    const StepLayout l = step_layout(d.N);
    StepParams prm{x, dt, A, B, C, D, state, y, d.T, d.H, d.P, d.G, d.N, l.L};
    if (d.dtype == SSD_BF16)
        return l.W == 4 ? launch_step_w<__nv_bfloat16, 4>(prm, l.K, d.b, s)
                        : launch_step_w<__nv_bfloat16, 1>(prm, l.K, d.b, s);
    return l.W == 4 ? launch_step_w<float, 4>(prm, l.K, d.b, s) : launch_step_w<float, 1>(prm, l.K, d.b, s);
}

}  // namespace ssd
