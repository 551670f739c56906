// Warp-specialized, persistent single-pass SSD forward for sm_100a.
//
// Same arithmetic as the fused mode of ssd_tc.cu ("Transformers are SSMs",
// Knowl 2, chunks chained through one L2-resident state buffer; the 128x128
// diagonal blocks of each chunk in the quadratic masked form, the lower
// off-diagonal 128-block through the state after the first tile), organised
// so that HBM traffic, tensor-core MMAs and CUDA-core work overlap:
//
//   warp 0      TMA producer: B/C tiles of a unit (one ring slot per 128-token
//               tile), x tile of each item (3-deep ring)
//   warp 1      TMEM owner and MMA issuer (one thread)
//   warp 2      per item: dt loads, cumulative sum of dt*A (log2 units) and the
//               per-token factors exp(cs_last - cs_i) dt_i and exp(cs_j)
//   warps 4-7   mask group: P = (C B^T) o mask from TMEM G into TMEM P (bf16,
//               the A operand of the Y product), and w o x into shared memory
//   warps 8-11  state/epilogue group: h as bf16 operand, h <- e h + S,
//               y = Y + exp(cs) R + D x to global memory, state hand-off
//
// Work: persistent CTAs take units (chunk c, batch row b, block of k heads of
// one group) round-robin in chunk-major order. An item is (unit, head, tile);
// a unit's items run head-major so that each head's state stays in registers
// between the tiles of its chunk.
//
// Tensor memory (512 columns): G of tile slot 0 / 1 (128 each), P (64, bf16
// pairs), Y (64), R (64), S (64).
//
// Every wait is bounded; a wait that gives up sets the error word and makes
// every role leave its loop, after which the CTA drains its MMAs and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sm100.cuh"
#include "ssd_internal.h"

namespace ssd {
namespace {

using namespace sm100;

constexpr int kTile = 128;
constexpr int kP = 64;
constexpr int kN = 128;
constexpr int kThreads = 384;
constexpr int kXStages = 3;
constexpr int kCsStages = 4;

constexpr uint32_t kAtom = kTile * 128;          // 16 KB: 128 rows of 128 bytes
constexpr uint32_t kBCSlot = 2 * (kN / 64) * kAtom;  // B and C of one tile: 64 KB
constexpr uint32_t kOffBC = 0;                   // 2 slots
constexpr uint32_t kOffX = kOffBC + 2 * kBCSlot;    // kXStages x 16 KB
constexpr uint32_t kOffWX = kOffX + kXStages * kAtom;
constexpr uint32_t kOffH = kOffWX + kAtom;
constexpr uint32_t kOffCs = kOffH + kN * 128;    // kCsStages x 4 arrays x 128 floats
constexpr uint32_t kCsSlot = 5 * kTile * 4;   // cs, dt, w, u, v (per item)
constexpr uint32_t kOffBar = kOffCs + kCsStages * kCsSlot;
constexpr uint32_t kSmemBytes = kOffBar + 512;

constexpr uint32_t kColG = 0;     // + 128 * slot
constexpr uint32_t kColP = 256;
constexpr uint32_t kColY = 320;
constexpr uint32_t kColR = 384;
constexpr uint32_t kColS = 448;

constexpr float kLog2e = 1.4426950408889634f;

struct Params {
    const __nv_bfloat16* x;
    const float* dt;
    const float* A;
    const float* D;
    const float* init;
    float* chain;
    __nv_bfloat16* y;
    int* flags;
    int* error;
    int64_t T, H, G, nc;
    int Q, kheads, batch, nunits;
};

struct Bars {
    uint64_t bc_full[2], bc_empty[2], g_full[2], g_empty[2];
    uint64_t x_full[kXStages], x_empty[kXStages];
    uint64_t cs_full[kCsStages], cs_empty[kCsStages];
    uint64_t p_full, p_empty, wx_full, wx_empty, h_full, h_empty, acc_full, acc_empty, fin;
    uint64_t chain_ok, pub;   // state hand-off inside the state/epilogue group
    uint32_t tmem;
    int abort;
};

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(h);
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded mbarrier wait (about 2 s) that also gives up as soon as another role
// aborted. try_wait itself suspends the thread for a while, so no sleep is added.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Bars* bs, int* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 0) {
            if (*(volatile int*)&bs->abort) return false;
            if (global_ns() - t0 > 2000000000ull) {
                *(volatile int*)&bs->abort = 1;
                atomicExch(err, 3);
                return false;
            }
        }
    }
}

// Same, called by all 32 lanes of a warp together: the outcome is made
// warp-uniform so that no lane leaves a loop its warp-mates stay in (the
// tcgen05.ld/st that follow are warp-collective).
__device__ __forceinline__ bool wait_bar_all(uint64_t* bar, uint32_t parity, Bars* bs, int* err) {
    const bool ok = wait_bar(bar, parity, bs, err);
    return __all_sync(0xffffffffu, ok);
}

// bf16 copy of the state as the B operand of C h^T: row n (one thread) holds
// h[0..63][n], 128-byte swizzled rows.
__device__ __forceinline__ void write_h_operand(uint8_t* sh, int n, const float (&hreg)[kP]) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
        *reinterpret_cast<uint4*>(sh + sw128_off(n, q)) =
            make_uint4(pack_bf16(hreg[8 * q], hreg[8 * q + 1]),
                       pack_bf16(hreg[8 * q + 2], hreg[8 * q + 3]),
                       pack_bf16(hreg[8 * q + 4], hreg[8 * q + 5]),
                       pack_bf16(hreg[8 * q + 6], hreg[8 * q + 7]));
}

struct Unit {
    int c, b, hb, nsub;
    int64_t tc0;
};
__device__ __forceinline__ Unit decode(const Params& p, int u) {
    const int nhb = (int)(p.H / p.kheads);
    Unit r;
    r.hb = u % nhb;
    r.b = (u / nhb) % p.batch;
    r.c = u / (nhb * p.batch);
    r.tc0 = (int64_t)r.c * p.Q;
    const int len = (int)min((int64_t)p.Q, p.T - r.tc0);
    r.nsub = (len + kTile - 1) / kTile;
    return r;
}

__global__ void __launch_bounds__(kThreads, 1)
    ssd_fused_ws_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_B,
                        const __grid_constant__ CUtensorMap tm_C, const Params prm) {
    extern __shared__ __align__(1024) uint8_t smem[];
    Bars* bs = reinterpret_cast<Bars*>(smem + kOffBar);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int* err = prm.error;

    if (tid == 0) {
        if ((smem_u32(smem) & 1023u) != 0) atomicExch(err, 4);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bs->bc_full[i], 1);
            mbar_init(&bs->bc_empty[i], 1);
            mbar_init(&bs->g_full[i], 1);
            mbar_init(&bs->g_empty[i], 128);
        }
        for (int i = 0; i < kXStages; ++i) {
            mbar_init(&bs->x_full[i], 1);
            mbar_init(&bs->x_empty[i], 1 + 128 + 128);
        }
        for (int i = 0; i < kCsStages; ++i) {
            mbar_init(&bs->cs_full[i], 32);
            mbar_init(&bs->cs_empty[i], 128 + 128);
        }
        mbar_init(&bs->p_full, 128);
        mbar_init(&bs->p_empty, 1);
        mbar_init(&bs->wx_full, 128);
        mbar_init(&bs->wx_empty, 1);
        mbar_init(&bs->h_full, 128);
        mbar_init(&bs->h_empty, 1);
        mbar_init(&bs->acc_full, 1);
        mbar_init(&bs->acc_empty, 128);
        mbar_init(&bs->fin, 1);
        mbar_init(&bs->chain_ok, 1);
        mbar_init(&bs->pub, 128);
        bs->abort = 0;
        fence_barrier_init();
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_B);
        prefetch_tmap(&tm_C);
    }
    if (warp == 1) tmem_alloc(&bs->tmem, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // the swizzled tiles need a 1024-byte aligned base; if not, skip all work
    // (error already set) but still release TMEM below
    const bool misaligned = (smem_u32(smem) & 1023u) != 0;
    const uint32_t tmem = bs->tmem;
    const int kh_n = prm.kheads;
    const int64_t T = prm.T, H = prm.H;

    if (misaligned) {
        // nothing
    } else if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int n = 0, m = 0;
            for (int u = blockIdx.x; u < prm.nunits; u += gridDim.x) {
                const Unit U = decode(prm, u);
                const int g = (int)((int64_t)U.hb * kh_n / (H / prm.G));
                for (int kh = 0; kh < kh_n; ++kh) {
                    const int h = U.hb * kh_n + kh;
                    for (int s = 0; s < U.nsub; ++s, ++n) {
                        if (kh == 0) {
                            // B and C of tile s, shared by every head of the unit
                            const int mm = m + s, sl = mm & 1;
                            if (!wait_bar(&bs->bc_empty[sl], ((mm >> 1) & 1) ^ 1, bs, err))
                                goto done;
                            mbar_arrive_expect_tx(&bs->bc_full[sl], kBCSlot);
                            uint8_t* base = smem + kOffBC + sl * kBCSlot;
                            for (int a = 0; a < kN / 64; ++a) {
                                tma_load_4d(base + a * kAtom, &tm_B, &bs->bc_full[sl], a * 64, g,
                                            (int)(U.tc0 + s * kTile), U.b);
                                tma_load_4d(base + kBCSlot / 2 + a * kAtom, &tm_C,
                                            &bs->bc_full[sl], a * 64, g,
                                            (int)(U.tc0 + s * kTile), U.b);
                            }
                        }
                        const int xs = n % kXStages;
                        if (!wait_bar(&bs->x_empty[xs], ((n / kXStages) & 1) ^ 1, bs, err))
                            goto done;
                        mbar_arrive_expect_tx(&bs->x_full[xs], kAtom);
                        tma_load_4d(smem + kOffX + xs * kAtom, &tm_x, &bs->x_full[xs], 0, h,
                                    (int)(U.tc0 + s * kTile), U.b);
                    }
                }
                m += U.nsub;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idG = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idS = idesc_bf16(128, kP, 1, 1);
            constexpr uint32_t idY = idesc_bf16(128, kP, 0, 1);
            int n = 0, m = 0;
            for (int u = blockIdx.x; u < prm.nunits; u += gridDim.x) {
                const Unit U = decode(prm, u);
                for (int kh = 0; kh < kh_n; ++kh) {
                    for (int s = 0; s < U.nsub; ++s, ++n) {
                        const int sl = (m + s) & 1, xs = n % kXStages;
                        if (kh == 0) {
                            // G = C B^T of tile s (diagonal block), shared by the unit's heads
                            const int ph = ((m + s) >> 1) & 1;
                            if (!wait_bar(&bs->bc_full[sl], ph, bs, err)) goto drain;
                            if (!wait_bar(&bs->g_empty[sl], ph ^ 1, bs, err)) goto drain;
                            tc_fence_after();
                            const uint32_t gB = smem_u32(smem + kOffBC + sl * kBCSlot);
                            const uint32_t gC = gB + kBCSlot / 2;
#pragma unroll
                            for (int kk = 0; kk < kN / 16; ++kk) {
                                const uint32_t off = (kk >> 2) * kAtom + (kk & 3) * 32;
                                mma_bf16(tmem + kColG + 128 * sl, sw128_desc(gC + off, 16, 1024),
                                         sw128_desc(gB + off, 16, 1024), idG, kk > 0);
                            }
                            mma_commit(&bs->g_full[sl]);
                        }
                        const uint32_t pn = n & 1;
                        if (!wait_bar(&bs->p_full, pn, bs, err)) goto drain;
                        if (!wait_bar(&bs->x_full[xs], (n / kXStages) & 1, bs, err)) goto drain;
                        if (!wait_bar(&bs->wx_full, pn, bs, err)) goto drain;
                        if (!wait_bar(&bs->h_full, pn, bs, err)) goto drain;
                        if (!wait_bar(&bs->acc_empty, pn ^ 1, bs, err)) goto drain;
                        tc_fence_after();
                        const uint32_t aB = smem_u32(smem + kOffBC + sl * kBCSlot);
                        const uint32_t aC = aB + kBCSlot / 2;
                        const uint32_t aX = smem_u32(smem + kOffX + xs * kAtom);
                        const uint32_t aWX = smem_u32(smem + kOffWX);
                        const uint32_t aH = smem_u32(smem + kOffH);
#pragma unroll
                        for (int kk = 0; kk < kTile / 16; ++kk)
                            mma_bf16_tmem_a(tmem + kColY, tmem + kColP + 8 * kk,
                                            sw128_desc(aX + kk * 2048, kAtom, 1024), idY, kk > 0);
#pragma unroll
                        for (int kk = 0; kk < kTile / 16; ++kk)
                            mma_bf16(tmem + kColS, sw128_desc(aB + kk * 2048, kAtom, 1024),
                                     sw128_desc(aWX + kk * 2048, kAtom, 1024), idS, kk > 0);
#pragma unroll
                        for (int kk = 0; kk < kN / 16; ++kk)
                            mma_bf16(tmem + kColR,
                                     sw128_desc(aC + (kk >> 2) * kAtom + (kk & 3) * 32, 16, 1024),
                                     sw128_desc(aH + kk * 2048, kAtom, 1024), idY, kk > 0);
                        mma_commit(&bs->p_empty);
                        mma_commit(&bs->wx_empty);
                        mma_commit(&bs->h_empty);
                        mma_commit(&bs->x_empty[xs]);
                        mma_commit(&bs->acc_full);
                        if (kh == kh_n - 1) mma_commit(&bs->bc_empty[sl]);
                    }
                }
                m += U.nsub;
            }
        drain:
            // every MMA issued so far is complete before TMEM is released
            mma_commit(&bs->fin);
            mbar_wait(&bs->fin, 0, 1u << 24);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ cumsum warp
        int n = 0;
        for (int u = blockIdx.x; u < prm.nunits; u += gridDim.x) {
            const Unit U = decode(prm, u);
            for (int kh = 0; kh < kh_n; ++kh) {
                const int h = U.hb * kh_n + kh;
                const float a2 = prm.A[h] * kLog2e;
                for (int s = 0; s < U.nsub; ++s, ++n) {
                    const int cb = n % kCsStages;
                    if (!wait_bar_all(&bs->cs_empty[cb], ((n / kCsStages) & 1) ^ 1, bs, err)) goto done;
                    const int64_t t0 = U.tc0 + (int64_t)s * kTile;
                    const int len = (int)min((int64_t)kTile, T - t0);
                    float dtv[4], v[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int t = lane * 4 + e;
                        dtv[e] = t < len ? __ldg(prm.dt + ((int64_t)U.b * T + t0 + t) * H + h) : 0.f;
                    }
                    float run = 0.f;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        run += dtv[e] * a2;
                        v[e] = run;
                    }
                    float incl = run;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const float o = __shfl_up_sync(0xffffffffu, incl, off);
                        if (lane >= off) incl += o;
                    }
                    const float excl = incl - run;
                    const float last = __shfl_sync(0xffffffffu, incl, 31);
                    float* cs = reinterpret_cast<float*>(smem + kOffCs + cb * kCsSlot);
                    float* dts = cs + kTile;
                    float* w = dts + kTile;
                    float* uu = w + kTile;
                    float* vv = uu + kTile;
                    // cs at the last row of this lane's 32-column block (lanes 8b..8b+7 hold block b)
                    const float cref = __shfl_sync(0xffffffffu, incl, (lane | 7));
                    float4 c4, d4, w4, u4, v4;
                    float* cp = &c4.x;
                    float* dp = &d4.x;
                    float* wp = &w4.x;
                    float* up = &u4.x;
                    float* vp = &v4.x;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float ce = excl + v[e];
                        cp[e] = ce;
                        dp[e] = dtv[e];
                        wp[e] = exp2f(last - ce) * dtv[e];
                        up[e] = exp2f(ce);
                        vp[e] = exp2f(cref - ce) * dtv[e];
                    }
                    reinterpret_cast<float4*>(cs)[lane] = c4;
                    reinterpret_cast<float4*>(dts)[lane] = d4;
                    reinterpret_cast<float4*>(w)[lane] = w4;
                    reinterpret_cast<float4*>(uu)[lane] = u4;
                    reinterpret_cast<float4*>(vv)[lane] = v4;
                    mbar_arrive(&bs->cs_full[cb]);
                }
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ mask group
        const int wq = warp - 4;
        const int j = tid - 128;  // row of the tile == TMEM lane
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        int n = 0, m = 0;
        for (int u = blockIdx.x; u < prm.nunits; u += gridDim.x) {
            const Unit U = decode(prm, u);
            for (int kh = 0; kh < kh_n; ++kh) {
                for (int s = 0; s < U.nsub; ++s, ++n) {
                    const int mm = m + s, sl = mm & 1;
                    const uint32_t pn = n & 1;
                    const int cb = n % kCsStages, xs = n % kXStages;
                    if (kh == 0 && !wait_bar_all(&bs->g_full[sl], (mm >> 1) & 1, bs, err)) goto done;
                    if (!wait_bar_all(&bs->cs_full[cb], (n / kCsStages) & 1, bs, err)) goto done;
                    if (!wait_bar_all(&bs->p_empty, pn ^ 1, bs, err)) goto done;
                    tc_fence_after();
                    __syncwarp();
                    const float* cs = reinterpret_cast<const float*>(smem + kOffCs + cb * kCsSlot);
                    const float* dts = cs + kTile;
                    const float* wv = dts + kTile;
                    const float* vv = wv + 2 * kTile;
                    const float csj = cs[j];
#pragma unroll 1
                    for (int blk = 0; blk < 4; ++blk) {
                        uint32_t pk[16];
                        if (blk > wq) {
#pragma unroll
                            for (int q = 0; q < 16; ++q) pk[q] = 0u;
                        } else if (blk < wq) {
                            // strictly below the diagonal block: every i < every j, and
                            // exp(cs_j - cs_i) = exp(cs_j - cs_ref) exp(cs_ref - cs_i) with
                            // ref the last row of column block blk; both factors are <= 1
                            float gv[32];
                            tmem_ld32(tmem + lane_base + kColG + 128 * sl + 32 * blk, gv);
                            const float uj = exp2f(csj - cs[32 * blk + 31]);
                            tmem_ld_wait();
#pragma unroll
                            for (int e4 = 0; e4 < 8; ++e4) {
                                const float4 v4 = reinterpret_cast<const float4*>(vv)[blk * 8 + e4];
                                pk[e4 * 2] = pack_bf16(gv[e4 * 4] * uj * v4.x, gv[e4 * 4 + 1] * uj * v4.y);
                                pk[e4 * 2 + 1] =
                                    pack_bf16(gv[e4 * 4 + 2] * uj * v4.z, gv[e4 * 4 + 3] * uj * v4.w);
                            }
                        } else {
                            float gv[32];
                            tmem_ld32(tmem + lane_base + kColG + 128 * sl + 32 * blk, gv);
                            tmem_ld_wait();
#pragma unroll
                            for (int e4 = 0; e4 < 8; ++e4) {
                                const float4 c4 = reinterpret_cast<const float4*>(cs)[blk * 8 + e4];
                                const float4 d4 = reinterpret_cast<const float4*>(dts)[blk * 8 + e4];
                                const int i0 = blk * 32 + e4 * 4;
                                const float m0 = exp2f(csj - c4.x) * d4.x;
                                const float m1 = exp2f(csj - c4.y) * d4.y;
                                const float m2 = exp2f(csj - c4.z) * d4.z;
                                const float m3 = exp2f(csj - c4.w) * d4.w;
                                const float p0 = (i0 <= j) ? gv[e4 * 4] * m0 : 0.f;
                                const float p1 = (i0 + 1 <= j) ? gv[e4 * 4 + 1] * m1 : 0.f;
                                const float p2 = (i0 + 2 <= j) ? gv[e4 * 4 + 2] * m2 : 0.f;
                                const float p3 = (i0 + 3 <= j) ? gv[e4 * 4 + 3] * m3 : 0.f;
                                pk[e4 * 2] = pack_bf16(p0, p1);
                                pk[e4 * 2 + 1] = pack_bf16(p2, p3);
                            }
                        }
                        tmem_st16(tmem + lane_base + kColP + 16 * blk, pk);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(&bs->p_full);
                    if (kh == kh_n - 1) mbar_arrive(&bs->g_empty[sl]);
                    // w o x, rows scaled by exp(cs_last - cs_i) dt_i
                    if (!wait_bar_all(&bs->x_full[xs], (n / kXStages) & 1, bs, err)) goto done;
                    if (!wait_bar_all(&bs->wx_empty, pn ^ 1, bs, err)) goto done;
                    {
                        const uint8_t* sx = smem + kOffX + xs * kAtom;
                        uint8_t* swx = smem + kOffWX;
                        const float w = wv[j];
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint4 xv = *reinterpret_cast<const uint4*>(sx + sw128_off(j, q));
                            const float2 a = unpack_bf16(xv.x), b = unpack_bf16(xv.y);
                            const float2 c2 = unpack_bf16(xv.z), d2 = unpack_bf16(xv.w);
                            *reinterpret_cast<uint4*>(swx + sw128_off(j, q)) = make_uint4(
                                pack_bf16(w * a.x, w * a.y), pack_bf16(w * b.x, w * b.y),
                                pack_bf16(w * c2.x, w * c2.y), pack_bf16(w * d2.x, w * d2.y));
                        }
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(&bs->wx_full);
                    mbar_arrive(&bs->x_empty[xs]);
                    mbar_arrive(&bs->cs_empty[cb]);
                }
            }
            m += U.nsub;
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ state / epilogue group
        const int wq = warp - 8;
        const int r = tid - 256;  // row j of the tile for outputs, n of the state
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        const int64_t PN = (int64_t)kP * kN;
        int n = 0, nchain = 0, npub = 0;
        for (int u = blockIdx.x; u < prm.nunits; u += gridDim.x) {
            const Unit U = decode(prm, u);
            for (int kh = 0; kh < kh_n; ++kh) {
                const int h = U.hb * kh_n + kh;
                const float D_h = prm.D ? prm.D[h] : 0.f;
                float hreg[kP];
                // state entering the chunk
                if (U.c == 0) {
                    const float* src = prm.init ? prm.init + ((int64_t)U.b * H + h) * PN + r : nullptr;
#pragma unroll
                    for (int p = 0; p < kP; ++p) hreg[p] = src ? __ldg(src + (int64_t)p * kN) : 0.f;
                } else {
                    if (r == 0) {
                        const int* f = prm.flags + (int64_t)U.b * H + h;
                        bool ok = false;
                        const uint64_t t0 = global_ns();
                        for (uint32_t it = 0;; ++it) {
                            if (ld_acquire(f) >= U.c) { ok = true; break; }
                            if ((it & 15) == 15 &&
                                (*(volatile int*)&bs->abort || global_ns() - t0 > 2000000000ull))
                                break;
                        }
                        if (!ok) {
                            *(volatile int*)&bs->abort = 1;
                            atomicExch(err, 1);
                        }
                        mbar_arrive(&bs->chain_ok);
                    }
                    if (!wait_bar_all(&bs->chain_ok, nchain & 1, bs, err)) goto done;
                    ++nchain;
                    if (*(volatile int*)&bs->abort) goto done;
                    __threadfence();
                    const float* src = prm.chain + ((int64_t)U.b * H + h) * PN + r;
#pragma unroll
                    for (int p = 0; p < kP; ++p) hreg[p] = __ldcg(src + (int64_t)p * kN);
                }
                for (int s = 0; s < U.nsub; ++s, ++n) {
                    const uint32_t pn = n & 1;
                    const int cb = n % kCsStages, xs = n % kXStages;
                    const int64_t t0 = U.tc0 + (int64_t)s * kTile;
                    const int len = (int)min((int64_t)kTile, T - t0);
                    // h as the B operand of C h^T (row n holds h[0..63][n]); for the first
                    // tile of the head here, for later tiles right after the state update
                    if (s == 0) {
                        if (!wait_bar_all(&bs->h_empty, pn ^ 1, bs, err)) goto done;
                        write_h_operand(smem + kOffH, r, hreg);
                        fence_proxy_async_smem();
                        mbar_arrive(&bs->h_full);
                    }
                    if (!wait_bar_all(&bs->cs_full[cb], (n / kCsStages) & 1, bs, err)) goto done;
                    if (!wait_bar_all(&bs->x_full[xs], (n / kXStages) & 1, bs, err)) goto done;
                    if (!wait_bar_all(&bs->acc_full, pn, bs, err)) goto done;
                    tc_fence_after();
                    __syncwarp();
                    const float* cs = reinterpret_cast<const float*>(smem + kOffCs + cb * kCsSlot);
                    const float* uu = cs + 3 * kTile;
                    const float e = uu[kTile - 1];   // exp(cs_last): decay over the whole tile
                    // h <- e h + S  (lane n holds S[n][0..63])
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float sv[32];
                        tmem_ld32(tmem + lane_base + kColS + 32 * half, sv);
                        tmem_ld_wait();
#pragma unroll
                        for (int p = 0; p < 32; ++p)
                            hreg[32 * half + p] = fmaf(e, hreg[32 * half + p], sv[p]);
                    }
                    if (s + 1 < U.nsub) {
                        // the R product of this item has completed (acc_full), so the
                        // operand buffer is free: stage the state entering the next tile
                        write_h_operand(smem + kOffH, r, hreg);
                        fence_proxy_async_smem();
                        mbar_arrive(&bs->h_full);
                    } else {
                        // hand the state of head h on to the next chunk before the epilogue
                        float* dst = prm.chain + ((int64_t)U.b * H + h) * PN + r;
#pragma unroll
                        for (int p = 0; p < kP; ++p) __stcg(dst + (int64_t)p * kN, hreg[p]);
                        __threadfence();
                        mbar_arrive(&bs->pub);
                        if (r == 0) {
                            if (wait_bar(&bs->pub, npub & 1, bs, err))
                                st_release(prm.flags + (int64_t)U.b * H + h, U.c + 1);
                        }
                        ++npub;
                        // lane 0 may have waited above: reconverge before warp-collective tcgen05.ld
                        __syncwarp();
                    }
                    // y_j = Y_j + exp(cs_j) R_j + D x_j
                    const float uj = uu[r];
                    const uint8_t* sx = smem + kOffX + xs * kAtom;
                    __nv_bfloat16* yrow = prm.y + (((int64_t)U.b * T + t0 + r) * H + h) * kP;
                    uint32_t pk[32];
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float yv[32], rv[32];
                        tmem_ld32(tmem + lane_base + kColY + 32 * half, yv);
                        tmem_ld32(tmem + lane_base + kColR + 32 * half, rv);
                        tmem_ld_wait();
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint4 xv =
                                *reinterpret_cast<const uint4*>(sx + sw128_off(r, 4 * half + q));
                            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                            for (int e2 = 0; e2 < 4; ++e2) {
                                const float2 xf = unpack_bf16(xw[e2]);
                                const int c0 = 8 * q + 2 * e2;
                                pk[16 * half + 4 * q + e2] =
                                    pack_bf16(fmaf(uj, rv[c0], yv[c0]) + D_h * xf.x,
                                              fmaf(uj, rv[c0 + 1], yv[c0 + 1]) + D_h * xf.y);
                            }
                        }
                    }
                    tc_fence_before();
                    mbar_arrive(&bs->acc_empty);
                    // the x tile was read through the generic proxy; the next TMA load into
                    // this slot is an async-proxy write, so order the reads before it
                    fence_proxy_async_smem();
                    mbar_arrive(&bs->x_empty[xs]);
                    mbar_arrive(&bs->cs_empty[cb]);
                    if (r < len) {
                        uint4* dst = reinterpret_cast<uint4*>(yrow);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                    }
                }
            }
        }
    }
done:
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

int g_num_sms = 0;

}  // namespace

cudaError_t launch_fused_ws(const Dims& d, const CUtensorMap* maps, const void* x, const float* dt,
                            const float* A, const float* D, const float* init, void* y,
                            float* chain, int* sync_ints, int kheads, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(sync_ints, 0, sizeof(int) * (size_t)(2 + d.b * d.H), st);
    if (e != cudaSuccess) return e;
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (g_num_sms <= 0) g_num_sms = 148;
    }
    Params prm = {};
    prm.x = (const __nv_bfloat16*)x;
    prm.dt = dt;
    prm.A = A;
    prm.D = D;
    prm.init = init;
    prm.chain = chain;
    prm.y = (__nv_bfloat16*)y;
    prm.error = sync_ints + 1;
    prm.flags = sync_ints + 2;
    prm.T = d.T;
    prm.H = d.H;
    prm.G = d.G;
    prm.nc = d.nc;
    prm.Q = (int)d.Q;
    prm.kheads = kheads;
    prm.batch = (int)d.b;
    prm.nunits = (int)(d.nc * d.b * (d.H / kheads));
    e = cudaFuncSetAttribute(ssd_fused_ws_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const int grid = prm.nunits < g_num_sms ? prm.nunits : g_num_sms;
    ssd_fused_ws_kernel<<<grid, kThreads, kSmemBytes, st>>>(maps[0], maps[1], maps[2], prm);
    return cudaGetLastError();
}

}  // namespace ssd
