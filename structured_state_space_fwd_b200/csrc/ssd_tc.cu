// Tensor-core (tcgen05 / TMEM / TMA) kernels of the SSD forward for sm_100a.
//
// One kernel template covers two steps of the block-decomposition algorithm
// ("Transformers are SSMs: Generalized Models and Efficient Algorithms Through
// Structured State Space Duality", Knowl 2) as separately callable steps:
//   kModeState  step 2, chunk states S_c = B_c^T (decayed X_c)
//   kModeScan   step 4, Y_c = (L o C B^T) dt X + decayed C h_c + D X, h_c given
//
// Work unit: (chunk c, batch row b, block of `kheads` heads of one group). The
// chunk's B and C tiles and its C B^T blocks (computed once on the tensor
// cores) serve every head of the block, since heads of a group share B and C
// (Knowl 7).
//
// Inside a chunk the kernel works in tiles of 128 tokens (the M of one tcgen05
// MMA). For a 256-token chunk, the two 128x128 diagonal blocks of the chunk's
// masked matrix L o C B^T are multiplied in the quadratic (masked attention)
// form, and the lower off-diagonal block through its rank-N factorisation:
// the state after the first tile carries it (the chunk matrix is
// N-semiseparable, Knowl 3), so the second tile sees the state entering it
// exactly as in Knowl 2's state passing. Per tile and head:
//   S   = B_t^T (w o X_t)       w_i = exp(cs_last - cs_i) dt_i          [tensor]
//   Y   = (G o mask) X_t        G = C_t B_t^T, mask_ji = exp(cs_j - cs_i) dt_i, i <= j
//   R   = C_t h^T               h = state entering the tile             [tensor]
//   y_j = Y_j + exp(cs_j) R_j + D x_j
//   h  <- exp(cs_last) h + S
// with cs the inclusive cumulative sum of dt*A inside the tile (log2 units).
//
// Shapes served: bf16 x/B/C/y, head dim 64, state dim 128, chunk 128 or 256.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "sm100.cuh"
#include "ssd_internal.h"

namespace ssd {
namespace {

using namespace sm100;

constexpr int kTile = 128;     // tokens per MMA tile
constexpr int kP = 64;         // head dim
constexpr int kN = 128;        // state dim
constexpr int kMaxSub = 2;     // tiles per chunk (chunk <= 256)
constexpr int kThreads = 128;  // one warpgroup: thread t <-> TMEM lane t

constexpr uint32_t kAtom = kTile * 128;             // one 128-row x 128-byte swizzle atom: 16 KB
constexpr uint32_t kBCBytes = (kN / 64) * kAtom;    // one tile of B (or C): 32 KB
constexpr uint32_t kOffB = 0;
constexpr uint32_t kOffC = kOffB + kMaxSub * kBCBytes;
constexpr uint32_t kOffX = kOffC + kMaxSub * kBCBytes;
constexpr uint32_t kOffP = kOffX + kAtom;
constexpr uint32_t kOffWX = kOffP + 2 * kAtom;
constexpr uint32_t kOffH = kOffWX + kAtom;
constexpr uint32_t kOffSmall = kOffH + kN * 128;   // h operand: N rows of 64 bf16
constexpr uint32_t kSmemBytes = kOffSmall + 4096 + 1024;  // small arrays + alignment slack

// TMEM columns (fp32, 128 lanes)
constexpr uint32_t kColG = 0;      // G of tile s at kColG + 128 s
constexpr uint32_t kColY = 256;
constexpr uint32_t kColR = 320;
constexpr uint32_t kColS = 384;
constexpr uint32_t kTmemCols = 512;

constexpr float kLog2e = 1.4426950408889634f;

enum Mode { kModeState = 0, kModeScan = 1 };

struct TcParams {
    const __nv_bfloat16* x;
    const float* dt;
    const float* D;
    const float* cs;          // step inputs [b,H,nc,Q] (state / scan modes)
    const float* entry;       // scan: states entering each chunk [b,nc,H,P,N]
    float* states_out;        // state mode: chunk states [b,nc,H,P,N]
    __nv_bfloat16* y;
    int* error;               // set when a bounded wait gives up (may be null)
    int64_t T, H, G, nc;
    int Q, kheads, batch;
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(h);
}

template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    ssd_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_B,
                  const __grid_constant__ CUtensorMap tm_C, const TcParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    uint8_t* sB = sm + kOffB;
    uint8_t* sC = sm + kOffC;
    uint8_t* sX = sm + kOffX;
    uint8_t* sP = sm + kOffP;
    uint8_t* sWX = sm + kOffWX;
    uint8_t* sH = sm + kOffH;
    float* s_cs = reinterpret_cast<float*>(sm + kOffSmall);  // [128] cumsum, log2 units
    float* s_dt = s_cs + kTile;                               // [128]
    float* s_wsum = s_dt + kTile;                             // [4]
    uint64_t* bar_bc = reinterpret_cast<uint64_t*>(s_wsum + 8);
    uint64_t* bar_x = bar_bc + 1;
    uint64_t* bar_mma = bar_bc + 2;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar_bc + 4);
    int* s_unit = reinterpret_cast<int*>(s_tmem + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    (void)lane;
    if (tid == 0) {
        mbar_init(bar_bc, 1);
        mbar_init(bar_x, 1);
        mbar_init(bar_mma, 1);
        fence_barrier_init();
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_B);
        if (kMode != kModeState) prefetch_tmap(&tm_C);
        *s_unit = (int)blockIdx.x;
    }
    if (warp == 0) tmem_alloc(s_tmem, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

    const int64_t T = prm.T, H = prm.H, nc = prm.nc;
    const int Q = prm.Q, kh_n = prm.kheads;
    const int nhb = (int)(H / kh_n);
    const int u = *s_unit;
    const int hb = u % nhb;
    const int bi = (u / nhb) % prm.batch;
    const int c = u / (nhb * prm.batch);
    const int g = (int)((int64_t)hb * kh_n / (H / prm.G));
    const int64_t tc0 = (int64_t)c * Q;
    const int len_c = (int)min((int64_t)Q, T - tc0);
    const int nsub = (len_c + kTile - 1) / kTile;
    uint32_t ph_x = 0, ph_mma = 0;

    // ---- B and C tiles of every 128-token tile of the chunk (shared by the heads)
    if (tid == 0) {
        const uint32_t per = (kMode == kModeState ? 1u : 2u) * kBCBytes;
        mbar_arrive_expect_tx(bar_bc, per * nsub);
        for (int s = 0; s < nsub; ++s) {
            for (int a = 0; a < kN / 64; ++a) {
                tma_load_4d(sB + s * kBCBytes + a * kAtom, &tm_B, bar_bc, a * 64, g,
                            (int)(tc0 + s * kTile), bi);
                if (kMode != kModeState)
                    tma_load_4d(sC + s * kBCBytes + a * kAtom, &tm_C, bar_bc, a * 64, g,
                                (int)(tc0 + s * kTile), bi);
            }
        }
    }
    if (!mbar_wait(bar_bc, 0)) {
        if (prm.error) atomicExch(prm.error, 2);
    }

    // ---- G_s = C_s B_s^T for each tile (diagonal blocks of C B^T)
    if (kMode != kModeState) {
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idG = idesc_bf16(128, 128, 0, 0);
            for (int s = 0; s < nsub; ++s) {
                const uint32_t aC = smem_u32(sC + s * kBCBytes), aB = smem_u32(sB + s * kBCBytes);
#pragma unroll
                for (int kk = 0; kk < kN / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                    mma_bf16(tmem + kColG + 128 * s, sw128_desc(aC + off, 16, 1024),
                             sw128_desc(aB + off, 16, 1024), idG, kk > 0);
                }
            }
            mma_commit(bar_mma);
        }
        mbar_wait(bar_mma, ph_mma);
        ph_mma ^= 1;
        tc_fence_after();
    }

    for (int kh = 0; kh < kh_n; ++kh) {
        const int h = hb * kh_n + kh;
        const float D_h = prm.D ? prm.D[h] : 0.f;
        const int64_t PN = (int64_t)kP * kN;
        float hreg[kP];  // thread n holds h[p][n] for p = 0..63

        // ---- state entering the chunk
        if (kMode == kModeState) {
#pragma unroll
            for (int p = 0; p < kP; ++p) hreg[p] = 0.f;
        } else {
            const float* src = prm.entry + (((int64_t)bi * nc + c) * H + h) * PN + tid;
#pragma unroll
            for (int p = 0; p < kP; ++p) hreg[p] = __ldg(src + (int64_t)p * kN);
        }

        for (int s = 0; s < nsub; ++s) {
            const int64_t t0 = tc0 + (int64_t)s * kTile;
            const int len = (int)min((int64_t)kTile, T - t0);
            // previous users of sX / sP / sWX / sH and of the TMEM accumulators are done;
            // the generic-proxy reads of sX are ordered before the next TMA write into it
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                mbar_arrive_expect_tx(bar_x, kAtom);
                tma_load_4d(sX, &tm_x, bar_x, 0, h, (int)t0, bi);
            }
            // ---- cumulative sum of dt*A over the tile (log2 units), inclusive
            float dtv = 0.f, v;
            // cs of the step interface: chunk-relative natural-log sums; rebase to the tile
            const float* csc = prm.cs + (((int64_t)bi * H + h) * nc + c) * Q + s * kTile;
            const float base = s > 0 ? csc[-1] : 0.f;
            if (tid < len) dtv = prm.dt[((int64_t)bi * T + t0 + tid) * H + h];
            v = (csc[min(tid, len - 1)] - base) * kLog2e;
            s_cs[tid] = v;
            s_dt[tid] = dtv;
            __syncthreads();
            const float cs_last = s_cs[kTile - 1];  // rows past the end repeat the last value
            if (!mbar_wait(bar_x, ph_x)) {
                if (prm.error) atomicExch(prm.error, 2);
            }
            ph_x ^= 1;

            // ---- masked diagonal block P = G o mask (bf16, K-major, 128B swizzle)
            if (kMode != kModeState) {
                const int j = tid;
                const float csj = s_cs[j];
                uint8_t* prow = sP;
#pragma unroll 1
                for (int cb = 0; cb < 4; ++cb) {
                    uint8_t* atom = prow + (cb >> 1) * kAtom;
                    const int chunk0 = (cb & 1) * 4;
                    if (cb > warp) {
                        const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            *reinterpret_cast<uint4*>(atom + sw128_off(j, chunk0 + q)) = z;
                        continue;
                    }
                    float gv[32];
                    tmem_ld32(tmem + lane_base + kColG + 128 * s + 32 * cb, gv);
                    tmem_ld_wait();
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int i0 = 32 * cb + e, i1 = i0 + 1;
                        const float m0 = exp2f(csj - s_cs[i0]) * s_dt[i0];
                        const float m1 = exp2f(csj - s_cs[i1]) * s_dt[i1];
                        const float p0 = (i0 <= j) ? gv[e] * m0 : 0.f;
                        const float p1 = (i1 <= j) ? gv[e + 1] * m1 : 0.f;
                        pk[e >> 1] = pack_bf16(p0, p1);
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<uint4*>(atom + sw128_off(j, chunk0 + q)) =
                            make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                }
            }
            // ---- w o X (rows scaled by exp(cs_last - cs_i) dt_i), same layout as X
            {
                const int i = tid;
                const float w = exp2f(cs_last - s_cs[i]) * s_dt[i];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint4 xv = *reinterpret_cast<const uint4*>(sX + sw128_off(i, q));
                    const float2 a = unpack_bf16(xv.x), b = unpack_bf16(xv.y);
                    const float2 cc = unpack_bf16(xv.z), d = unpack_bf16(xv.w);
                    *reinterpret_cast<uint4*>(sWX + sw128_off(i, q)) =
                        make_uint4(pack_bf16(w * a.x, w * a.y), pack_bf16(w * b.x, w * b.y),
                                   pack_bf16(w * cc.x, w * cc.y), pack_bf16(w * d.x, w * d.y));
                }
            }
            // ---- h (bf16) as the B operand of C h^T: row n holds h[0..63][n]
            if (kMode != kModeState) {
                const int n = tid;
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    *reinterpret_cast<uint4*>(sH + sw128_off(n, q)) =
                        make_uint4(pack_bf16(hreg[8 * q], hreg[8 * q + 1]),
                                   pack_bf16(hreg[8 * q + 2], hreg[8 * q + 3]),
                                   pack_bf16(hreg[8 * q + 4], hreg[8 * q + 5]),
                                   pack_bf16(hreg[8 * q + 6], hreg[8 * q + 7]));
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();

            // ---- tensor-core products of this tile
            if (tid == 0) {
                tc_fence_after();
                const uint32_t aB = smem_u32(sB + s * kBCBytes);
                const uint32_t aWX = smem_u32(sWX);
                constexpr uint32_t idS = idesc_bf16(128, kP, 1, 1);
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk)
                    mma_bf16(tmem + kColS, sw128_desc(aB + kk * 2048, kAtom, 1024),
                             sw128_desc(aWX + kk * 2048, kAtom, 1024), idS, kk > 0);
                if (kMode != kModeState) {
                    const uint32_t aP = smem_u32(sP), aX = smem_u32(sX);
                    const uint32_t aC = smem_u32(sC + s * kBCBytes), aH = smem_u32(sH);
                    constexpr uint32_t idY = idesc_bf16(128, kP, 0, 1);
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk)
                        mma_bf16(tmem + kColY,
                                 sw128_desc(aP + (kk >> 2) * kAtom + (kk & 3) * 32, 16, 1024),
                                 sw128_desc(aX + kk * 2048, kAtom, 1024), idY, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < kN / 16; ++kk)
                        mma_bf16(tmem + kColR,
                                 sw128_desc(aC + (kk >> 2) * kAtom + (kk & 3) * 32, 16, 1024),
                                 sw128_desc(aH + kk * 2048, kAtom, 1024), idY, kk > 0);
                }
                mma_commit(bar_mma);
            }
            if (!mbar_wait(bar_mma, ph_mma)) {
                if (prm.error) atomicExch(prm.error, 2);
            }
            ph_mma ^= 1;
            tc_fence_after();

            // ---- output rows: y_j = Y_j + exp(cs_j) R_j + D x_j
            if (kMode != kModeState) {
                const int j = tid;
                const float uj = exp2f(s_cs[j]);
                __nv_bfloat16* yrow = prm.y + (((int64_t)bi * T + t0 + j) * H + h) * kP;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float yv[32], rv[32];
                    tmem_ld32(tmem + lane_base + kColY + 32 * half, yv);
                    tmem_ld32(tmem + lane_base + kColR + 32 * half, rv);
                    tmem_ld_wait();
                    uint32_t pk[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 xv =
                            *reinterpret_cast<const uint4*>(sX + sw128_off(j, 4 * half + q));
                        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 xf = unpack_bf16(xw[e]);
                            const int c0 = 8 * q + 2 * e;
                            pk[4 * q + e] = pack_bf16(yv[c0] + uj * rv[c0] + D_h * xf.x,
                                                      yv[c0 + 1] + uj * rv[c0 + 1] + D_h * xf.y);
                        }
                    }
                    if (j < len) {
                        uint4* dst = reinterpret_cast<uint4*>(yrow + 32 * half);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                    }
                }
            }
            // ---- state after the tile: h <- exp(cs_last) h + S  (thread n, lane n)
            {
                const float e = exp2f(cs_last);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float sv[32];
                    tmem_ld32(tmem + lane_base + kColS + 32 * half, sv);
                    tmem_ld_wait();
#pragma unroll
                    for (int p = 0; p < 32; ++p)
                        hreg[32 * half + p] = fmaf(e, hreg[32 * half + p], sv[p]);
                }
            }
        }

        // ---- hand the state on
        if (kMode == kModeState) {
            float* dst = prm.states_out + (((int64_t)bi * nc + c) * H + h) * PN + tid;
#pragma unroll
            for (int p = 0; p < kP; ++p) dst[(int64_t)p * kN] = hreg[p];
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 4-D bf16 map over [d3][d2][d1][d0] (d0 innermost), box {64, 1, 128, 1}, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t d3,
              uint32_t box_rows = kTile) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {d0, d1, d2, d3};
    const cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
    const cuuint32_t box[4] = {64, 1, box_rows, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int pick_kheads(int64_t heads_per_group) {
    for (int k = 4; k > 1; --k)
        if (heads_per_group % k == 0) return k;
    return 1;
}

bool make_tc_maps(const Dims& d, const void* x, const void* B, const void* C, const void* y,
                  CUtensorMap* maps) {
    return make_map(&maps[0], x, d.P, d.H, d.T, d.b) && make_map(&maps[1], B, d.N, d.G, d.T, d.b) &&
           make_map(&maps[2], C ? C : B, d.N, d.G, d.T, d.b) &&
           make_map(&maps[3], y ? y : x, d.P, d.H, d.T, d.b, 32);
}

namespace {

template <int kMode>
cudaError_t launch_tc(const Dims& d, TcParams prm, const void* x, const void* B, const void* C,
                      cudaStream_t st) {
    CUtensorMap mx, mB, mC;
    if (!make_map(&mx, x, d.P, d.H, d.T, d.b) || !make_map(&mB, B, d.N, d.G, d.T, d.b) ||
        !make_map(&mC, C ? C : B, d.N, d.G, d.T, d.b))
        return cudaErrorInvalidValue;
    prm.T = d.T;
    prm.H = d.H;
    prm.G = d.G;
    prm.nc = d.nc;
    prm.Q = (int)d.Q;
    prm.batch = (int)d.b;
    prm.kheads = pick_kheads(d.H / d.G);
    const int64_t units = d.nc * d.b * (d.H / prm.kheads);
    auto k = ssd_tc_kernel<kMode>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    k<<<(unsigned)units, kThreads, kSmemBytes, st>>>(mx, mB, mC, prm);
    return cudaGetLastError();
}

}  // namespace

bool tma_available() { return encode_fn() != nullptr; }

bool tc_supported(const Dims& d) {
    return d.dtype == SSD_BF16 && d.P == kP && d.N == kN && (d.Q == 128 || d.Q == 256) &&
           d.T <= 0x7fffffffLL && d.b <= 0x7fffffffLL && d.nc * d.b * d.H < 0x7fffffffLL &&
           encode_fn() != nullptr;
}

cudaError_t launch_chunk_state_tc(const Dims& d, const void* x, const float* dt, const void* B,
                                  const float* cs, float* states, cudaStream_t st) {
    TcParams prm = {};
    prm.x = (const __nv_bfloat16*)x;
    prm.dt = dt;
    prm.cs = cs;
    prm.states_out = states;
    return launch_tc<kModeState>(d, prm, x, B, nullptr, st);
}

cudaError_t launch_chunk_scan_tc(const Dims& d, const void* x, const float* dt, const void* B,
                                 const void* C, const float* D, const float* cs,
                                 const float* entry, void* y, cudaStream_t st) {
    TcParams prm = {};
    prm.x = (const __nv_bfloat16*)x;
    prm.dt = dt;
    prm.D = D;
    prm.cs = cs;
    prm.entry = entry;
    prm.y = (__nv_bfloat16*)y;
    return launch_tc<kModeScan>(d, prm, x, B, C, st);
}

}  // namespace ssd
