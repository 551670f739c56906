// Gate and normalisation after the SSD layer ("Transformers are SSMs:
// Generalized Models and Efficient Algorithms Through Structured State Space
// Duality", Knowl 6, step 4 of the Mamba-2 block): the layer output y is gated
// elementwise by SiLU(z), then RMS-normalised before the output projection.
// Per token and group of `gs` contiguous channels (channels = H * P, as y is
// laid out):
//
//     v_c   = y_c * z_c / (1 + exp(-z_c))
//     out_c = v_c / sqrt(mean_group(v^2) + eps) * weight_c
//
// HBM-bound: y and z are read once and out written once (6 bytes per channel
// in bf16). A group is handled by TPG threads (4..256) of a 256-thread CTA;
// each thread keeps up to kMaxVec 16-byte vectors of v in registers between
// the sum of squares and the scaled write, and groups larger than that are
// re-read (from L2) for the write.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ssd_internal.h"

namespace ssd {
namespace {

constexpr int kGateThreads = 256;
constexpr int kMaxVec = 4;

__device__ __forceinline__ void load_vec(const float* p, float (&v)[4]) {
    const float4 q = *reinterpret_cast<const float4*>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}
__device__ __forceinline__ void load_vec(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 q = *reinterpret_cast<const uint4*>(p);
    const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void load_vec(const float* p, float (&v)[1]) { v[0] = *p; }
__device__ __forceinline__ void load_vec(const __nv_bfloat16* p, float (&v)[1]) { v[0] = __bfloat162float(*p); }

__device__ __forceinline__ void store_vec(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store_vec(__nv_bfloat16* p, const float (&v)[8]) {
    uint32_t u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        u[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(u[0], u[1], u[2], u[3]);
}
__device__ __forceinline__ void store_vec(float* p, const float (&v)[1]) { *p = v[0]; }
__device__ __forceinline__ void store_vec(__nv_bfloat16* p, const float (&v)[1]) { *p = __float2bfloat16_rn(v[0]); }

// SiLU through the special-function unit (__expf, __fdividef): a few ulp, far
// inside the fp32 bar at the gate's range, and 0 for very negative z (the
// divisor overflows to inf). The accurate expf and IEEE division cost about
// 40 instructions per element and made the pass 0.43 of the copy peak
// instead of 0.57 (measured).
template <int VW>
__device__ __forceinline__ void gate(const float (&y)[VW], const float (&z)[VW], float (&v)[VW]) {
#pragma unroll
    for (int i = 0; i < VW; ++i) v[i] = y[i] * __fdividef(z[i], 1.f + __expf(-z[i]));
}

// E: storage type; VW: elements per vector (16 bytes, or 1 when the group size is
// not a multiple of 16 bytes); TPG: threads per group. Registers are capped so
// that 5 CTAs fit on an SM (measured faster than 4 with no spills).
template <typename E, int VW, int TPG>
__global__ void __launch_bounds__(kGateThreads, 5) gated_rmsnorm_kernel(
    const E* __restrict__ y, const E* __restrict__ z, const float* __restrict__ w, E* __restrict__ out,
    int64_t ngroups_total, int64_t groups_per_row, int64_t gs, float eps) {
    constexpr int GPB = kGateThreads / TPG;            // groups per CTA
    constexpr int WPG = TPG / 32 > 0 ? TPG / 32 : 1;   // warps per group
    __shared__ float red[kGateThreads / 32];
    const int tg = threadIdx.x % TPG;                  // thread within its group
    const int slot = threadIdx.x / TPG;
    const int64_t grp = (int64_t)blockIdx.x * GPB + slot;
    const bool live = grp < ngroups_total;
    const int64_t base = live ? grp * gs : 0;           // rows are contiguous groups
    const int64_t wbase = live ? (grp % groups_per_row) * gs : 0;
    const int64_t nvec = gs / VW;

    float v[kMaxVec][VW];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i) {
        const int64_t idx = tg + (int64_t)i * TPG;
        if (live && idx < nvec) {
            float a[VW], b[VW];
            load_vec(y + base + idx * VW, a);
            load_vec(z + base + idx * VW, b);
            gate<VW>(a, b, v[i]);
#pragma unroll
            for (int e = 0; e < VW; ++e) ss = fmaf(v[i][e], v[i][e], ss);
        }
    }
    for (int64_t idx = tg + (int64_t)kMaxVec * TPG; live && idx < nvec; idx += TPG) {
        float a[VW], b[VW], g[VW];
        load_vec(y + base + idx * VW, a);
        load_vec(z + base + idx * VW, b);
        gate<VW>(a, b, g);
#pragma unroll
        for (int e = 0; e < VW; ++e) ss = fmaf(g[e], g[e], ss);
    }
        // sum over the group's threads: within the warp (or the group's lanes of it, which
    // are aligned), then across its warps
#pragma unroll
    for (int off = (TPG < 32 ? TPG : 32) / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if constexpr (WPG > 1) {
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
        __syncthreads();
        ss = 0.f;
#pragma unroll
        for (int k = 0; k < WPG; ++k) ss += red[slot * WPG + k];
    }
    if (!live) return;
    const float r = rsqrtf(ss / (float)gs + eps);
#pragma unroll
    for (int i = 0; i < kMaxVec; ++i) {
        const int64_t idx = tg + (int64_t)i * TPG;
        if (idx < nvec) {
            float o[VW];
#pragma unroll
            for (int e = 0; e < VW; ++e) o[e] = v[i][e] * r * w[wbase + idx * VW + e];
            store_vec(out + base + idx * VW, o);
        }
    }
    for (int64_t idx = tg + (int64_t)kMaxVec * TPG; idx < nvec; idx += TPG) {
        float a[VW], b[VW], g[VW], o[VW];
        load_vec(y + base + idx * VW, a);
        load_vec(z + base + idx * VW, b);
        gate<VW>(a, b, g);
#pragma unroll
        for (int e = 0; e < VW; ++e) o[e] = g[e] * r * w[wbase + idx * VW + e];
        store_vec(out + base + idx * VW, o);
    }
}

template <typename E, int VW>
cudaError_t launch_gate_vw(const E* y, const E* z, const float* w, E* out, int64_t rows, int64_t C,
                           int64_t gs, float eps, cudaStream_t st) {
    const int64_t nvec = gs / VW;
    const int64_t groups = rows * (C / gs);
    // threads per group: enough for kMaxVec vectors each, at least 4 (a small group
    // shares its warp with others rather than leaving lanes idle)
    int tpg = 4;
    while (tpg < kGateThreads && (int64_t)tpg * kMaxVec < nvec) tpg <<= 1;
    const int64_t gpb = kGateThreads / tpg;
    const unsigned grid = (unsigned)((groups + gpb - 1) / gpb);
    const int64_t gpr = C / gs;
    switch (tpg) {
        case 4: gated_rmsnorm_kernel<E, VW, 4><<<grid, kGateThreads, 0, st>>>(y, z, w, out, groups, gpr, gs, eps); break;
        case 8: gated_rmsnorm_kernel<E, VW, 8><<<grid, kGateThreads, 0, st>>>(y, z, w, out, groups, gpr, gs, eps); break;
        case 16: gated_rmsnorm_kernel<E, VW, 16><<<grid, kGateThreads, 0, st>>>(y, z, w, out, groups, gpr, gs, eps); break;
        case 32: gated_rmsnorm_kernel<E, VW, 32><<<grid, kGateThreads, 0, st>>>(y, z, w, out, groups, gpr, gs, eps); break;
        case 64: gated_rmsnorm_kernel<E, VW, 64><<<grid, kGateThreads, 0, st>>>(y, z, w, out, groups, gpr, gs, eps); break;
        case 128: gated_rmsnorm_kernel<E, VW, 128><<<grid, kGateThreads, 0, st>>>(y, z, w, out, groups, gpr, gs, eps); break;
        default: gated_rmsnorm_kernel<E, VW, 256><<<grid, kGateThreads, 0, st>>>(y, z, w, out, groups, gpr, gs, eps); break;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gated_rmsnorm(const Dims& d, const void* y, const void* z, const float* w,
                                 int64_t group_size, float eps, void* out, cudaStream_t st) {
    const int64_t rows = d.b * d.T, C = d.H * d.P;
    if (rows == 0) return cudaSuccess;
    if (d.dtype == SSD_BF16) {
        auto* yy = static_cast<const __nv_bfloat16*>(y);
        auto* zz = static_cast<const __nv_bfloat16*>(z);
        auto* oo = static_cast<__nv_bfloat16*>(out);
        return group_size % 8 == 0 ? launch_gate_vw<__nv_bfloat16, 8>(yy, zz, w, oo, rows, C, group_size, eps, st)
                                   : launch_gate_vw<__nv_bfloat16, 1>(yy, zz, w, oo, rows, C, group_size, eps, st);
    }
    auto* yy = static_cast<const float*>(y);
    auto* zz = static_cast<const float*>(z);
    auto* oo = static_cast<float*>(out);
    return group_size % 4 == 0 ? launch_gate_vw<float, 4>(yy, zz, w, oo, rows, C, group_size, eps, st)
                               : launch_gate_vw<float, 1>(yy, zz, w, oo, rows, C, group_size, eps, st);
}

}  // namespace ssd
