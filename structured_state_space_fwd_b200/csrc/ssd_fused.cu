// Warp-specialized, persistent single-pass SSD forward for sm_100a.
//
// Same arithmetic as the fused mode of ssd_tc.cu ("Transformers are SSMs",
// Knowl 2, chunks chained through one L2-resident state buffer; the 128x128
// diagonal blocks of each chunk in the quadratic masked form, the lower
// off-diagonal 128-block through the state after the first tile), organised
// so that HBM traffic, tensor-core MMAs and CUDA-core work overlap:
//
//   warp 0      TMA producer: B/C tiles of a unit (one ring slot per 128-token
//               tile), x tile of each item (2-deep ring)
//   warp 1      TMEM owner and MMA issuer (one thread)
//   warp 2      per item: dt loads, cumulative sum of dt*A (log2 units) and the
//               per-token factors exp(cs_last - cs_i) dt_i and exp(cs_j)
//   warp 3      lane 0 releases chain flags
//   warps 4-7   mask group: P = (C B^T) o mask from TMEM G into TMEM P (bf16,
//               the A operand of the Y product), and w o x into shared memory
//   warps 8-15  state/epilogue group, two warps per TMEM lane quarter, each
//               owning half of the head dim: drains S, Y, R from TMEM, then
//               h <- e h + S, the bf16 state operand, w o x of the next item,
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
constexpr int kThreads = 512;
constexpr int kXStages = 3;
constexpr int kWXStages = 1;
constexpr int kCsStages = 4;
constexpr int kPubStages = 4;

constexpr uint32_t kAtom = kTile * 128;          // 16 KB: 128 rows of 128 bytes
constexpr uint32_t kBCSlot = 2 * (kN / 64) * kAtom;  // B and C of one tile: 64 KB
constexpr uint32_t kOffBC = 0;                   // 2 slots
constexpr uint32_t kOffX = kOffBC + 2 * kBCSlot;    // kXStages x 16 KB
constexpr uint32_t kOffWX = kOffX + kXStages * kAtom;
constexpr uint32_t kOffH = kOffWX + kWXStages * kAtom;
constexpr uint32_t kOffCs = kOffH + kN * 128;    // kCsStages x 4 arrays x 128 floats
constexpr uint32_t kCsSlot = 6 * kTile * 4;   // cs, dt, w, u, v (per item), then D_h
constexpr uint32_t kOffBar = kOffCs + kCsStages * kCsSlot;
constexpr uint32_t kSmemBytes = kOffBar + 512;

constexpr uint32_t kColG = 0;     // + 128 * slot
constexpr uint32_t kColP = 256;
constexpr uint32_t kColY = 320;
constexpr uint32_t kColR = 384;
constexpr uint32_t kColS = 448;

constexpr float kLog2e = 1.4426950408889634f;
// Widest cs range (log2 units) of a 32-row diagonal block for which the masked
// product is formed as exp2(cs_j - cs_e) * exp2(cs_e - cs_i): both factors then
// stay within 2^+-64, far from fp32 overflow for any finite G.
constexpr float kFactorRangeLog2 = 64.f;

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
    uint64_t wx_full[kWXStages], wx_empty[kWXStages];
    uint64_t p_full, p_empty, h_full, h_empty, fin;
    uint64_t sr_full, s_empty;    // S and R done; S drained by the state group
    uint64_t y_full, ry_empty;    // Y done; R and Y drained by the state group
    uint64_t chain_ok;                          // chain flag observed (state group)
    uint64_t pub_full[kPubStages], pub_empty[kPubStages];  // state stored / flag released
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
__device__ __forceinline__ uint32_t pack_bf16(float2 v) { return pack_bf16(v.x, v.y); }
// packed fp32 pairs (one instruction for two lanes of arithmetic)
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// A suspend-time hint on try_wait measured slower here (the woken thread
// resumes later than a spinning one notices), so waits spin by default.
#ifndef SSD_WAIT_HINT_NS
#define SSD_WAIT_HINT_NS 0u
#endif
__device__ __forceinline__ bool try_wait(uint64_t* bar, uint32_t parity) {
#if SSD_WAIT_HINT_NS > 0
    return mbar_try_wait_hint(bar, parity, SSD_WAIT_HINT_NS);
#else
    return mbar_try_wait(bar, parity);
#endif
}

// Bounded mbarrier wait (about 2 s) that also gives up once another role
// aborted (checked every 16 polls).
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Bars* bs, int* err) {
    if (try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (try_wait(bar, parity)) return true;
        if ((i & 15) == 0) {
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

// Half of a row of the bf16 state operand: thread (n, half) writes h[32 half + i][n],
// i < 32, into chunks 4 half .. 4 half + 3 of row n.
__device__ __forceinline__ void write_h_half(uint8_t* sh, int n, int half, const float (&hh)[32]) {
#pragma unroll
    for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(sh + sw128_off(n, 4 * half + c)) =
            make_uint4(pack_bf16(hh[8 * c], hh[8 * c + 1]), pack_bf16(hh[8 * c + 2], hh[8 * c + 3]),
                       pack_bf16(hh[8 * c + 4], hh[8 * c + 5]), pack_bf16(hh[8 * c + 6], hh[8 * c + 7]));
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
                        const __grid_constant__ CUtensorMap tm_C,
                        const __grid_constant__ CUtensorMap tm_y, const Params prm) {
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
            // Y product (commit) + state group twice (w o x, then the skip term x)
            mbar_init(&bs->x_empty[i], 1 + 256 + 256);
        }
        for (int i = 0; i < kCsStages; ++i) {
            mbar_init(&bs->cs_full[i], 32);
            mbar_init(&bs->cs_empty[i], 128 + 256);
        }
        mbar_init(&bs->p_full, 128);
        mbar_init(&bs->p_empty, 1);
        for (int i = 0; i < kWXStages; ++i) {
            mbar_init(&bs->wx_full[i], 256);
            mbar_init(&bs->wx_empty[i], 1);   // S product (commit)
        }
        mbar_init(&bs->h_full, 256);
        mbar_init(&bs->h_empty, 1);
        mbar_init(&bs->sr_full, 1);
        mbar_init(&bs->s_empty, 256);
        mbar_init(&bs->y_full, 1);
        mbar_init(&bs->ry_empty, 256);
        mbar_init(&bs->fin, 1);
        mbar_init(&bs->chain_ok, 1);
        for (int i = 0; i < kPubStages; ++i) {
            mbar_init(&bs->pub_full[i], 256);
            mbar_init(&bs->pub_empty[i], 1);
        }
        bs->abort = 0;
        fence_barrier_init();
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_B);
        prefetch_tmap(&tm_C);
        prefetch_tmap(&tm_y);
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
                            const uint64_t dGA = sw128_desc(gB + kBCSlot / 2, 16, 1024);
                            const uint64_t dGB = sw128_desc(gB, 16, 1024);
#pragma unroll
                            for (int kk = 0; kk < kN / 16; ++kk) {
                                // start address advances by (kk/4) atoms + (kk%4) x 32 bytes
                                const uint64_t off = (uint64_t)(((kk >> 2) * kAtom + (kk & 3) * 32) >> 4);
                                mma_bf16(tmem + kColG + 128 * sl, dGA + off, dGB + off, idG, kk > 0);
                            }
                            mma_commit(&bs->g_full[sl]);
                        }
                        const uint32_t pn = n & 1;
                        const int ws = n % kWXStages;
                        // S = B^T (w o x) and R = C h^T first: the state update waits on them
                        if (!wait_bar(&bs->wx_full[ws], (n / kWXStages) & 1, bs, err)) goto drain;
                        if (!wait_bar(&bs->h_full, pn, bs, err)) goto drain;
                        if (!wait_bar(&bs->s_empty, pn ^ 1, bs, err)) goto drain;
                        if (!wait_bar(&bs->ry_empty, pn ^ 1, bs, err)) goto drain;
                        tc_fence_after();
                        const uint32_t aB = smem_u32(smem + kOffBC + sl * kBCSlot);
                        const uint64_t dSA = sw128_desc(aB, kAtom, 1024);
                        const uint64_t dSB = sw128_desc(smem_u32(smem + kOffWX + ws * kAtom), kAtom, 1024);
                        const uint64_t dRA = sw128_desc(aB + kBCSlot / 2, 16, 1024);
                        const uint64_t dRB = sw128_desc(smem_u32(smem + kOffH), kAtom, 1024);
#pragma unroll
                        for (int kk = 0; kk < kTile / 16; ++kk) {
                            const uint64_t rows = (uint64_t)(kk * (2048 >> 4));   // 16 rows of 128 B
                            const uint64_t kofs = (uint64_t)(((kk >> 2) * kAtom + (kk & 3) * 32) >> 4);
                            mma_bf16(tmem + kColS, dSA + rows, dSB + rows, idS, kk > 0);
                            mma_bf16(tmem + kColR, dRA + kofs, dRB + rows, idY, kk > 0);
                        }
                        mma_commit(&bs->wx_empty[ws]);
                        mma_commit(&bs->h_empty);
                        mma_commit(&bs->sr_full);
                        // Y = P x (P straight from TMEM)
                        if (!wait_bar(&bs->p_full, pn, bs, err)) goto drain;
                        if (!wait_bar(&bs->x_full[xs], (n / kXStages) & 1, bs, err)) goto drain;
                        tc_fence_after();
                        const uint64_t dXB = sw128_desc(smem_u32(smem + kOffX + xs * kAtom), kAtom, 1024);
#pragma unroll
                        for (int kk = 0; kk < kTile / 16; ++kk)
                            mma_bf16_tmem_a(tmem + kColY, tmem + kColP + 8 * kk,
                                            dXB + (uint64_t)(kk * (2048 >> 4)), idY, kk > 0);
                        mma_commit(&bs->p_empty);
                        mma_commit(&bs->x_empty[xs]);
                        mma_commit(&bs->y_full);
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
                const float d_h = prm.D ? prm.D[h] : 0.f;
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
                    if (lane == 0) vv[kTile] = d_h;
                    __syncwarp();
                    mbar_arrive(&bs->cs_full[cb]);
                }
            }
        }
    } else if (warp == 3) {
        if (lane == 0) {
            // ---------------------------------------------------------- chain publisher
            // The state group stores a head's state and arrives on pub_full; this lane
            // then makes those stores visible GPU-wide (one fence, cumulative over the
            // stores ordered before the barrier) and releases the head's chain flag.
            int np = 0;
            for (int u = blockIdx.x; u < prm.nunits; u += gridDim.x) {
                const Unit U = decode(prm, u);
                for (int kh = 0; kh < kh_n; ++kh, ++np) {
                    const int h = U.hb * kh_n + kh;
                    const int ps = np % kPubStages;
                    if (!wait_bar(&bs->pub_full[ps], (np / kPubStages) & 1, bs, err)) goto done;
                    __threadfence();
                    st_release(prm.flags + (int64_t)U.b * H + h, U.c + 1);
                    mbar_arrive(&bs->pub_empty[ps]);
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
                    const int cb = n % kCsStages;
                    if (!wait_bar_all(&bs->cs_full[cb], (n / kCsStages) & 1, bs, err)) goto done;
                    const float* cs = reinterpret_cast<const float*>(smem + kOffCs + cb * kCsSlot);
                    const float* dts = cs + kTile;
                    const float* vv = dts + 3 * kTile;
                    // masked diagonal block P = G o mask into TMEM
                    if (kh == 0 && !wait_bar_all(&bs->g_full[sl], (mm >> 1) & 1, bs, err)) goto done;
                    if (!wait_bar_all(&bs->p_empty, pn ^ 1, bs, err)) goto done;
                    tc_fence_after();
                    __syncwarp();
                    const float csj = cs[j];
                    const int jj = j & 31;   // row within this warp's diagonal block
#pragma unroll 1
                    for (int blk = 0; blk < 4; ++blk) {
                        uint32_t pk[16];
                        if (blk > wq) {
#pragma unroll
                            for (int q = 0; q < 16; ++q) pk[q] = 0u;
                        } else {
                            float gv[32];
                            tmem_ld32(tmem + lane_base + kColG + 128 * sl + 32 * blk, gv);
                            // exp(cs_j - cs_i) dt_i = exp(cs_j - cs_e) * v_i with e the last row of
                            // column block blk and v_i = exp(cs_e - cs_i) dt_i (<= dt_i). Below the
                            // diagonal block the first factor is <= 1 too; on it, it is >= 1 and
                            // bounded by the block's own cs range, which decides whether the
                            // factored form is safe in fp32 or the exponent is taken per element.
                            const float ce = cs[32 * blk + 31];
                            const float a = exp2f(csj - ce);
                            const bool exact = blk == wq && cs[32 * blk] - ce > kFactorRangeLog2;
                            const float2 a2 = make_float2(a, a);
                            tmem_ld_wait();
                            if (blk < wq) {
#pragma unroll
                                for (int e4 = 0; e4 < 8; ++e4) {
                                    const float4 v4 = reinterpret_cast<const float4*>(vv)[blk * 8 + e4];
                                    pk[e4 * 2] = pack_bf16(mul2(make_float2(gv[e4 * 4], gv[e4 * 4 + 1]),
                                                                mul2(make_float2(v4.x, v4.y), a2)));
                                    pk[e4 * 2 + 1] = pack_bf16(mul2(make_float2(gv[e4 * 4 + 2], gv[e4 * 4 + 3]),
                                                                    mul2(make_float2(v4.z, v4.w), a2)));
                                }
                            } else if (!exact) {
#pragma unroll
                                for (int e4 = 0; e4 < 8; ++e4) {
                                    const float4 v4 = reinterpret_cast<const float4*>(vv)[blk * 8 + e4];
                                    float2 p01 = mul2(make_float2(gv[e4 * 4], gv[e4 * 4 + 1]),
                                                      mul2(make_float2(v4.x, v4.y), a2));
                                    float2 p23 = mul2(make_float2(gv[e4 * 4 + 2], gv[e4 * 4 + 3]),
                                                      mul2(make_float2(v4.z, v4.w), a2));
                                    const int i0 = e4 * 4;   // causal mask: column i kept while i <= row
                                    p01.x = i0 <= jj ? p01.x : 0.f;
                                    p01.y = i0 + 1 <= jj ? p01.y : 0.f;
                                    p23.x = i0 + 2 <= jj ? p23.x : 0.f;
                                    p23.y = i0 + 3 <= jj ? p23.y : 0.f;
                                    pk[e4 * 2] = pack_bf16(p01);
                                    pk[e4 * 2 + 1] = pack_bf16(p23);
                                }
                            } else {
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
                        }
                        tmem_st16(tmem + lane_base + kColP + 16 * blk, pk);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(&bs->p_full);
                    if (kh == kh_n - 1) mbar_arrive(&bs->g_empty[sl]);
                    mbar_arrive(&bs->cs_empty[cb]);
                }
            }
            m += U.nsub;
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ state / epilogue group
        // Iteration n finishes item n and prepares item n+1: drain S_n as soon as it is
        // done (so the next S and R can follow Y on the tensor pipe), update the state,
        // stage the next state operand (next tile of this head, or publish this head and
        // enter the next one), build w o x of item n+1, then drain Y_n and R_n into y_n.
        const int q = warp & 3;                 // TMEM lane quarter
        const int ph = (warp - 8) >> 2;         // half of the head dim this warp owns
        const int r = q * 32 + lane;            // tile row for outputs, state index n
        const bool leader = (warp == 8 && lane == 0);
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const int64_t PN = (int64_t)kP * kN;
        int nchain = 0, npub = 0;
        float hreg[32];  // h[32 ph + i][r] of the head being processed
        // State entering chunk U.c of head h into hreg, and its bf16 copy as the B operand
        // of the first tile's C h^T (item `item`). Returns false on abort.
        auto enter_head = [&](const Unit& U, int h, int item) -> bool {
            if (U.c == 0) {
                const float* src =
                    prm.init ? prm.init + ((int64_t)U.b * H + h) * PN + (int64_t)(32 * ph) * kN + r : nullptr;
#pragma unroll
                for (int i = 0; i < 32; ++i) hreg[i] = src ? __ldg(src + (int64_t)i * kN) : 0.f;
            } else {
                if (leader) {
                    const int* f = prm.flags + (int64_t)U.b * H + h;
                    bool ok = false;
                    const uint64_t t0 = global_ns();
                    for (uint32_t it = 0;; ++it) {
                        if (ld_acquire(f) >= U.c) { ok = true; break; }
                        if (it >= 8) __nanosleep(32);
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
                if (!wait_bar_all(&bs->chain_ok, nchain & 1, bs, err)) return false;
                ++nchain;
                if (*(volatile int*)&bs->abort) return false;
                __threadfence();
                const float* src = prm.chain + ((int64_t)U.b * H + h) * PN + (int64_t)(32 * ph) * kN + r;
#pragma unroll
                for (int i = 0; i < 32; ++i) hreg[i] = __ldcg(src + (int64_t)i * kN);
            }
            if (!wait_bar_all(&bs->h_empty, (item & 1) ^ 1, bs, err)) return false;
            write_h_half(smem + kOffH, r, ph, hreg);
            fence_proxy_async_smem();
            mbar_arrive(&bs->h_full);
            return true;
        };
        // items in the order every role walks them: nx is the next one (unit, head,
        // tile), cur the one being finished (batch row, head, first token, last tile
        // of its chunk or not)
        int nx_u = blockIdx.x, nx_kh = 0, nx_s = 0;
        bool nx_ok = nx_u < prm.nunits;
        Unit nxU{};
        if (nx_ok) nxU = decode(prm, nx_u);
        bool cur_ok = false, cur_last = false;
        int cur_b = 0, cur_h = 0;
        int64_t cur_t0 = 0;
        for (int n = -1; cur_ok || nx_ok; ++n) {
            const int nn = n < 0 ? 0 : n;
            const uint32_t pn = nn & 1;
            const int cb = nn % kCsStages, xs = nn % kXStages;
            const float* cs = reinterpret_cast<const float*>(smem + kOffCs + cb * kCsSlot);
            const float* uu = cs + 3 * kTile;
            if (cur_ok) {
                if (!wait_bar_all(&bs->cs_full[cb], (nn / kCsStages) & 1, bs, err)) goto done;
                if (!wait_bar_all(&bs->sr_full, pn, bs, err)) goto done;
                tc_fence_after();
                __syncwarp();
                // drain S (this warp's 32 columns), release it, update the state
                {
                    const float e = uu[kTile - 1];   // exp(cs_last): decay over the whole tile
                    const float2 e2 = make_float2(e, e);
                    float sv[32];
                    tmem_ld32(tmem + lane_base + kColS + 32 * ph, sv);
                    tmem_ld_wait();
                    tc_fence_before();
                    mbar_arrive(&bs->s_empty);
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const float2 t = fma2(e2, make_float2(hreg[i], hreg[i + 1]),
                                              make_float2(sv[i], sv[i + 1]));
                        hreg[i] = t.x;
                        hreg[i + 1] = t.y;
                    }
                }
                if (!cur_last) {
                    // R of this item is complete, so the operand buffer is free:
                    // stage the state entering the next tile
                    write_h_half(smem + kOffH, r, ph, hreg);
                    fence_proxy_async_smem();
                    mbar_arrive(&bs->h_full);
                } else {
                    // hand the state of head h on (flag released by warp 3)
                    const int ps = npub % kPubStages;
                    if (!wait_bar_all(&bs->pub_empty[ps], ((npub / kPubStages) & 1) ^ 1, bs, err))
                        goto done;
                    float* dst = prm.chain + ((int64_t)cur_b * H + cur_h) * PN + (int64_t)(32 * ph) * kN + r;
#pragma unroll
                    for (int i = 0; i < 32; ++i) __stcg(dst + (int64_t)i * kN, hreg[i]);
                    mbar_arrive(&bs->pub_full[ps]);
                    ++npub;
                }
            }
            if (nx_ok) {
                const int item = n + 1;
                // a new head: its entering state, so the next item's products can start
                if (nx_s == 0 && !enter_head(nxU, nxU.hb * kh_n + nx_kh, item)) goto done;
                // w o x of the next item: row r of its x tile scaled by
                // w_r = exp(cs_last - cs_r) dt_r, this warp's half of the head dim
                const int xs1 = item % kXStages, ws1 = item % kWXStages, cb1 = item % kCsStages;
                if (!wait_bar_all(&bs->cs_full[cb1], (item / kCsStages) & 1, bs, err)) goto done;
                if (!wait_bar_all(&bs->x_full[xs1], (item / kXStages) & 1, bs, err)) goto done;
                if (!wait_bar_all(&bs->wx_empty[ws1], ((item / kWXStages) & 1) ^ 1, bs, err)) goto done;
                const float w = reinterpret_cast<const float*>(smem + kOffCs + cb1 * kCsSlot)[2 * kTile + r];
                const float2 w2 = make_float2(w, w);
                const uint8_t* sx = smem + kOffX + xs1 * kAtom;
                uint8_t* swx = smem + kOffWX + ws1 * kAtom;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t off = sw128_off(r, 4 * ph + c);
                    const uint4 xv = *reinterpret_cast<const uint4*>(sx + off);
                    *reinterpret_cast<uint4*>(swx + off) =
                        make_uint4(pack_bf16(mul2(w2, unpack_bf16(xv.x))), pack_bf16(mul2(w2, unpack_bf16(xv.y))),
                                   pack_bf16(mul2(w2, unpack_bf16(xv.z))), pack_bf16(mul2(w2, unpack_bf16(xv.w))));
                }
                fence_proxy_async_smem();
                mbar_arrive(&bs->wx_full[ws1]);
                mbar_arrive(&bs->x_empty[xs1]);
            }
            if (cur_ok) {
                // R and Y (this warp's 32 columns) in two halves of 16:
                // y_j = Y_j + exp(cs_j) R_j + D x_j, this thread's bytes of row r
                if (!wait_bar_all(&bs->y_full, pn, bs, err)) goto done;
                tc_fence_after();
                __syncwarp();
                const float uj = uu[r];
                const float D_h = uu[2 * kTile];
                const float2 u2 = make_float2(uj, uj), d2 = make_float2(D_h, D_h);
                const uint8_t* sx = smem + kOffX + xs * kAtom;
                uint4* dst = reinterpret_cast<uint4*>(
                    prm.y + (((int64_t)cur_b * T + cur_t0 + r) * H + cur_h) * kP + 32 * ph);
                const bool valid = cur_t0 + r < T;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float yv[16], rv[16];
                    tmem_ld16(tmem + lane_base + kColY + 32 * ph + 16 * hf, yv);
                    tmem_ld16(tmem + lane_base + kColR + 32 * ph + 16 * hf, rv);
                    uint4 xq[2];
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        xq[c] = *reinterpret_cast<const uint4*>(sx + sw128_off(r, 4 * ph + 2 * hf + c));
                    tmem_ld_wait();
                    if (hf == 1) {
                        tc_fence_before();
                        mbar_arrive(&bs->ry_empty);
                        // generic-proxy reads of the x slot are done before the next
                        // TMA load into it
                        fence_proxy_async_smem();
                        mbar_arrive(&bs->x_empty[xs]);
                    }
                    uint4 out[2];
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const uint32_t xw[4] = {xq[c].x, xq[c].y, xq[c].z, xq[c].w};
                        uint32_t o[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const int i0 = 8 * c + 2 * e2;
                            const float2 t = fma2(u2, make_float2(rv[i0], rv[i0 + 1]),
                                                  make_float2(yv[i0], yv[i0 + 1]));
                            o[e2] = pack_bf16(fma2(d2, unpack_bf16(xw[e2]), t));
                        }
                        out[c] = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                    if (valid) {
                        dst[2 * hf] = out[0];
                        dst[2 * hf + 1] = out[1];
                    }
                }
                mbar_arrive(&bs->cs_empty[cb]);
            }
            // step the item iterator
            cur_ok = nx_ok;
            if (nx_ok) {
                cur_b = nxU.b;
                cur_h = nxU.hb * kh_n + nx_kh;
                cur_t0 = nxU.tc0 + (int64_t)nx_s * kTile;
                cur_last = nx_s + 1 >= nxU.nsub;
                if (++nx_s >= nxU.nsub) {
                    nx_s = 0;
                    if (++nx_kh >= kh_n) {
                        nx_kh = 0;
                        nx_u += gridDim.x;
                        nx_ok = nx_u < prm.nunits;
                        if (nx_ok) nxU = decode(prm, nx_u);
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
    ssd_fused_ws_kernel<<<grid, kThreads, kSmemBytes, st>>>(maps[0], maps[1], maps[2], maps[3], prm);
    return cudaGetLastError();
}

}  // namespace ssd
