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
// the sum of squares and the scaled write. Groups that fit that way run on a
// persistent grid that loads a CTA's next groups while it reduces and writes
// the current ones; larger groups are re-read (from L2) for the write.
#include <algorithm>
#include <type_traits>

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

// SiLU through the special-function unit. fp32 data: __expf and __fdividef, a
// few ulp, far inside the fp32 bar at the gate's range, and 0 for very negative
// z (the divisor overflows to inf); the accurate expf and IEEE division cost
// about 40 instructions per element and made the pass 0.43 of the copy peak
// instead of 0.57 (measured). bf16 data: z sigmoid(z) = z (1 + tanh(z / 2)) / 2,
// one tanh.approx (relative error about 2^-11, below bf16's rounding of the
// output), one special-function operation per element instead of two.
__device__ __forceinline__ float silu_tanh(float z) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
    return 0.5f * z * (1.f + t);
}
template <int VW, bool kTanh>
__device__ __forceinline__ void gate(const float (&y)[VW], const float (&z)[VW], float (&v)[VW]) {
#pragma unroll
    for (int i = 0; i < VW; ++i) v[i] = kTanh ? y[i] * silu_tanh(z[i]) : y[i] * __fdividef(z[i], 1.f + __expf(-z[i]));
}

// E: storage type; VW: elements per vector (16 bytes, or 1 when the group size is
// not a multiple of 16 bytes); TPG: threads per group. Registers are capped so
// that 5 CTAs fit on an SM (measured faster than 4 with no spills).
// The raw 16-byte vector (or one element) of a load, converted after it lands.
template <typename E, int VW>
struct RawVec {
    using T = uint4;
};
template <typename E>
struct RawVec<E, 1> {
    using T = E;
};
__device__ __forceinline__ void unpack(const uint4& q, float (&v)[8]) {
    const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void unpack(const uint4& q, float (&v)[4]) {
    v[0] = __uint_as_float(q.x); v[1] = __uint_as_float(q.y); v[2] = __uint_as_float(q.z); v[3] = __uint_as_float(q.w);
}
__device__ __forceinline__ void unpack(const float& q, float (&v)[1]) { v[0] = q; }
__device__ __forceinline__ void unpack(const __nv_bfloat16& q, float (&v)[1]) { v[0] = __bfloat162float(q); }
template <int VW>
__device__ __forceinline__ void load_w(const float* p, float (&v)[VW]) {
    if constexpr (VW == 1) {
        v[0] = *p;
    } else {
#pragma unroll
        for (int i = 0; i < VW; i += 4) {
            const float4 q = *reinterpret_cast<const float4*>(p + i);
            v[i] = q.x; v[i + 1] = q.y; v[i + 2] = q.z; v[i + 3] = q.w;
        }
    }
}

// Groups of at most kMaxVec * TPG vectors: each CTA walks the groups
// blockIdx.x * GPB + slot + k * gridDim.x * GPB. The loads of a CTA's next groups
// are issued before the current ones are reduced and written, so they are in
// flight across the reduction's barrier and the stores.
// CTAs per SM of the pipelined kernel (registers for the current and the next
// groups' vectors without spills; measured: one group per CTA 93 µs with 3 CTAs
// per SM against 99 with 2, groups of 64 channels 105 µs with 2 against 114 with 3)
__host__ __device__ constexpr int pipe_ctas(int tpg) { return tpg >= 128 ? 3 : 2; }
template <typename E, int VW, int TPG>
__global__ void __launch_bounds__(kGateThreads, pipe_ctas(TPG)) gated_rmsnorm_pipelined_kernel(
    const E* __restrict__ y, const E* __restrict__ z, const float* __restrict__ w, E* __restrict__ out,
    int64_t ngroups_total, int64_t groups_per_row, int64_t gs, float eps) {
    using Raw = typename RawVec<E, VW>::T;
    constexpr bool kBf16 = std::is_same<E, __nv_bfloat16>::value;
    constexpr int GPB = kGateThreads / TPG;
    constexpr int WPG = TPG / 32 > 0 ? TPG / 32 : 1;
    __shared__ float red[2][kGateThreads / 32];
    const int tg = threadIdx.x % TPG;
    const int slot = threadIdx.x / TPG;
    const int64_t nvec = gs / VW;
    const int64_t stride = (int64_t)gridDim.x * GPB;
    Raw ry[kMaxVec], rz[kMaxVec];
    auto issue = [&](int64_t grp) {
        const bool live = grp < ngroups_total;
        const int64_t base = live ? grp * gs : 0;
#pragma unroll
        for (int i = 0; i < kMaxVec; ++i) {
            const int64_t idx = tg + (int64_t)i * TPG;
            if (live && idx < nvec) {
                ry[i] = __ldcs(reinterpret_cast<const Raw*>(y + base + idx * VW));
                rz[i] = __ldcs(reinterpret_cast<const Raw*>(z + base + idx * VW));
            }
        }
    };
    int64_t grp = (int64_t)blockIdx.x * GPB + slot;
    issue(grp);
    for (int it = 0; (int64_t)blockIdx.x * GPB + (int64_t)it * stride < ngroups_total; ++it, grp += stride) {
        const bool live = grp < ngroups_total;
        float v[kMaxVec][VW];
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxVec; ++i) {
            const int64_t idx = tg + (int64_t)i * TPG;
            if (live && idx < nvec) {
                float a[VW], b[VW];
                unpack(ry[i], a);
                unpack(rz[i], b);
                gate<VW, kBf16>(a, b, v[i]);
#pragma unroll
                for (int e = 0; e < VW; ++e) ss = fmaf(v[i][e], v[i][e], ss);
            }
        }
        issue(grp + stride);
#pragma unroll
        for (int off = (TPG < 32 ? TPG : 32) / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if constexpr (WPG > 1) {
            if ((threadIdx.x & 31) == 0) red[it & 1][threadIdx.x >> 5] = ss;
            __syncthreads();
            ss = 0.f;
#pragma unroll
            for (int k = 0; k < WPG; ++k) ss += red[it & 1][slot * WPG + k];
        }
        if (live) {
            const int64_t base = grp * gs;
            const int64_t wbase = (grp % groups_per_row) * gs;
            const float r = rsqrtf(ss / (float)gs + eps);
#pragma unroll
            for (int i = 0; i < kMaxVec; ++i) {
                const int64_t idx = tg + (int64_t)i * TPG;
                if (idx < nvec) {
                    float o[VW], wv[VW];
                    load_w<VW>(w + wbase + idx * VW, wv);
#pragma unroll
                    for (int e = 0; e < VW; ++e) o[e] = v[i][e] * r * wv[e];
                    store_vec(out + base + idx * VW, o);
                }
            }
        }
    }
}

template <typename E, int VW, int TPG>
__global__ void __launch_bounds__(kGateThreads, 5) gated_rmsnorm_kernel(
    const E* __restrict__ y, const E* __restrict__ z, const float* __restrict__ w, E* __restrict__ out,
    int64_t ngroups_total, int64_t groups_per_row, int64_t gs, float eps) {
    constexpr bool kBf16 = std::is_same<E, __nv_bfloat16>::value;
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
            gate<VW, kBf16>(a, b, v[i]);
#pragma unroll
            for (int e = 0; e < VW; ++e) ss = fmaf(v[i][e], v[i][e], ss);
        }
    }
    for (int64_t idx = tg + (int64_t)kMaxVec * TPG; live && idx < nvec; idx += TPG) {
        float a[VW], b[VW], g[VW];
        load_vec(y + base + idx * VW, a);
        load_vec(z + base + idx * VW, b);
        gate<VW, kBf16>(a, b, g);
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
        gate<VW, kBf16>(a, b, g);
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
    if ((int64_t)tpg * kMaxVec >= nvec) {
        // persistent: pipe_ctas(tpg) CTAs per SM, each over every grid-th block of groups
        int dev = 0, sms = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const unsigned pg = (unsigned)std::min<int64_t>(grid, (int64_t)(sms > 0 ? sms : 148) * pipe_ctas(tpg));
        switch (tpg) {
            case 4: gated_rmsnorm_pipelined_kernel<E, VW, 4><<<pg, kGateThreads, 0, st>>>(y, z, w, out, groups, gpr, gs, eps); break;
            case 8: gated_rmsnorm_pipelined_kernel<E, VW, 8><<<pg, kGateThreads, 0, st>>>(y, z, w, out, groups, gpr, gs, eps); break;
            case 16: gated_rmsnorm_pipelined_kernel<E, VW, 16><<<pg, kGateThreads, 0, st>>>(y, z, w, out, groups, gpr, gs, eps); break;
            case 32: gated_rmsnorm_pipelined_kernel<E, VW, 32><<<pg, kGateThreads, 0, st>>>(y, z, w, out, groups, gpr, gs, eps); break;
            case 64: gated_rmsnorm_pipelined_kernel<E, VW, 64><<<pg, kGateThreads, 0, st>>>(y, z, w, out, groups, gpr, gs, eps); break;
            case 128: gated_rmsnorm_pipelined_kernel<E, VW, 128><<<pg, kGateThreads, 0, st>>>(y, z, w, out, groups, gpr, gs, eps); break;
            default: gated_rmsnorm_pipelined_kernel<E, VW, 256><<<pg, kGateThreads, 0, st>>>(y, z, w, out, groups, gpr, gs, eps); break;
        }
        return cudaGetLastError();
    }
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
