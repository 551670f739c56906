// Warp-specialized, persistent single-pass SSD forward for sm_100a.
//
// "Transformers are SSMs" (Knowl 2, Knowl 7) with the chunk equal to one
// 128-token tile: per tile the diagonal block in the quadratic masked form,
// everything before the tile through the state entering it. Roles:
//
//   warp 0      TMA producer: B/C tile of each unit (2-slot ring), x tile of
//               each item (3-slot ring)
//   warp 1      TMEM owner and MMA issuer (one thread)
//   warp 2      per item: dt loads, cumulative sum of dt*A (log2 units) and the
//               per-token factors
//   warp 3      lane 0 releases chain flags
//   warps 4-7   mask group: P = (C B^T) o L into TMEM (bf16, A operand of Y)
//   warps 8-15  state/epilogue group, two warps per TMEM lane quarter, each
//               owning half of the head dim: the head's state after the tile
//               out of TMEM onto the chain, the next item's operands (bf16
//               entering state for C h^T, exp(cs_last) h preloaded into the S
//               accumulator, w o x), then y = Y + exp(cs) R + D x
//
// Work: persistent CTAs take units (tile t, batch row b, block of k heads of
// one group) round-robin in tile-major order; an item is (unit, head), so
// consecutive items never share a state. The state of (b, h) after tile t
// goes to tile t+1 through one L2-resident buffer and a release/acquire flag.
//
// Tensor memory (512 columns): G (128), P (64, bf16 pairs), S (64), R 2 x 64,
// Y 2 x 64: R and Y are double-buffered so an item's products do not wait for
// the previous item's epilogue.
//
// Every wait is bounded; a wait that gives up sets the error word and makes
// every role leave its loop, after which the CTA drains its MMAs and exits.
#include <cstdlib>

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
constexpr int kCsStages = 4;
constexpr int kPubStages = 4;

constexpr uint32_t kAtom = kTile * 128;          // 16 KB: 128 rows of 128 bytes
constexpr uint32_t kBCSlot = 2 * (kN / 64) * kAtom;  // B and C of one tile: 64 KB
constexpr uint32_t kOffBC = 0;                   // 2 slots
constexpr uint32_t kOffX = kOffBC + 2 * kBCSlot;    // kXStages x 16 KB
constexpr uint32_t kOffWX = kOffX + kXStages * kAtom;
constexpr uint32_t kOffH = kOffWX + kAtom;
constexpr uint32_t kOffCs = kOffH + kN * 128;    // kCsStages slots
constexpr uint32_t kCsSlot = 7 * kTile * 4;   // cs, dt, w, u, v, u' (per token), then D_h, unit flag
constexpr uint32_t kOffBar = kOffCs + kCsStages * kCsSlot;
constexpr uint32_t kSmemBytes = kOffBar + 512;

constexpr uint32_t kColG = 0;
constexpr uint32_t kColP = 128;
constexpr uint32_t kColS = 192;
constexpr uint32_t kColR = 256;   // + 64 * buffer
constexpr uint32_t kColY = 384;   // + 64 * buffer

constexpr float kLog2e = 1.4426950408889634f;
// Widest cs range (log2 units) of a 32-row diagonal block for which the masked
// product is formed as exp2(cs_j - cs_e) * exp2(cs_e - cs_i): both factors then
// stay within 2^+-64, far from fp32 overflow for any finite G.
constexpr float kFactorRangeLog2 = 64.f;
// Widest decay over one tile (log2 units) for which the tile's masked product is
// formed head-independently, Y' = tril(C B^T) (w o x) with y = exp2(cs - cs_last) Y':
// both exp2(cs_last - cs) dt (in w o x, bf16) and its inverse stay inside the
// normal fp32/bf16 exponent range with a wide margin.
constexpr float kSharedMaskRangeLog2 = 96.f;

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
    int64_t T;
    int H, G, kheads, batch, nunits;
    int stall;   // test hook: chain flags are awaited at a value never reached
};

struct Bars {
    uint64_t bc_full[2], bc_empty[2];
    uint64_t g_full, g_empty;
    uint64_t x_full[kXStages], x_empty[kXStages];
    uint64_t cs_full[kCsStages], cs_empty[kCsStages];
    uint64_t wx_full, wx_empty;
    uint64_t p_full, p_empty;
    uint64_t h_full, h_empty;     // state operand and S preload written / operand read
    uint64_t s_full;              // S complete: the head's state after the tile
    uint64_t y_full[2], ry_empty[2];
    uint64_t y_staged[8];         // a lane quarter's y rows written (warp 12+q to 8+q), per item parity
    uint64_t pub_full[kPubStages], pub_empty[kPubStages];  // state stored / flag released
    uint64_t fin;
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

#ifndef SSD_IDLE_SLEEP_NS
#define SSD_IDLE_SLEEP_NS 100
#endif
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
__device__ __noinline__ bool wait_bar_slow(uint64_t* bar, uint32_t parity, Bars* bs, int* err) {
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
// Fast path inline, the polling loop shared by every call site (one copy in the
// instruction caches).
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Bars* bs, int* err) {
    if (try_wait(bar, parity)) return true;
    return wait_bar_slow(bar, parity, bs, err);
}


// Same for roles that run ahead of their consumers (TMA producer, cumsum warp,
// chain publisher): between polls the thread sleeps, so that its warp leaves the
// issue slots of its scheduler to the compute warps that share it.
__device__ __noinline__ bool wait_bar_idle_slow(uint64_t* bar, uint32_t parity, Bars* bs, int* err) {
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        __nanosleep(SSD_IDLE_SLEEP_NS);
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
__device__ __forceinline__ bool wait_bar_idle(uint64_t* bar, uint32_t parity, Bars* bs, int* err) {
    if (try_wait(bar, parity)) return true;
    return wait_bar_idle_slow(bar, parity, bs, err);
}


#ifdef SSD_MMA_IDLE
#define MMA_WAIT wait_bar_idle
#else
#define MMA_WAIT wait_bar
#endif

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

// 2^x on the special-function unit (a few ulp; results below 2^-126 flush to
// zero, i.e. decays too small to matter).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct Unit {
    int t, b, hb;     // tile, batch row, head block
    int64_t t0;       // first token of the tile
};
__device__ __forceinline__ Unit decode(const Params& p, int u) {
    const int nhb = p.H / p.kheads;
    Unit r;
    r.hb = u % nhb;
    r.b = (u / nhb) % p.batch;
    r.t = u / (nhb * p.batch);
    r.t0 = (int64_t)r.t * kTile;
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
            mbar_init(&bs->y_full[i], 1);
            mbar_init(&bs->ry_empty[i], 256);
        }
        for (int i = 0; i < 8; ++i) mbar_init(&bs->y_staged[i], 32);
        mbar_init(&bs->g_full, 1);
        mbar_init(&bs->g_empty, 128);
        for (int i = 0; i < kXStages; ++i) {
            mbar_init(&bs->x_full[i], 1);
            // Y product (commit) + mask group (w o x) + the 4 lanes that store y from it
            mbar_init(&bs->x_empty[i], 1 + 128 + 4);
        }
        for (int i = 0; i < kCsStages; ++i) {
            mbar_init(&bs->cs_full[i], 32);
            mbar_init(&bs->cs_empty[i], 128 + 256);
        }
        mbar_init(&bs->wx_full, 128);
        mbar_init(&bs->wx_empty, 1);
        mbar_init(&bs->p_full, 128);
        mbar_init(&bs->p_empty, 1);
        mbar_init(&bs->h_full, 256);
        mbar_init(&bs->h_empty, 1);
        mbar_init(&bs->s_full, 1);
        for (int i = 0; i < kPubStages; ++i) {
            mbar_init(&bs->pub_full[i], 256);
            mbar_init(&bs->pub_empty[i], 1);
        }
        mbar_init(&bs->fin, 1);
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
    const int64_t T = prm.T;
    const int H = prm.H;

    if (misaligned) {
        // nothing
    } else if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int n = 0, m = 0;    // x tiles and B/C tiles issued
            for (int u = blockIdx.x; u < prm.nunits; u += gridDim.x) {
                const Unit U = decode(prm, u);
                const int g = U.hb * kh_n / (H / prm.G);
                // B and C of the tile, shared by every head of the unit
                const int sl = m & 1;
                if (!wait_bar_idle(&bs->bc_empty[sl], ((m >> 1) & 1) ^ 1, bs, err)) goto pdrain;
                mbar_arrive_expect_tx(&bs->bc_full[sl], kBCSlot);
                uint8_t* base = smem + kOffBC + sl * kBCSlot;
                for (int a = 0; a < kN / 64; ++a) {
                    tma_load_4d(base + a * kAtom, &tm_B, &bs->bc_full[sl], a * 64, g, (int)U.t0, U.b);
                    tma_load_4d(base + kBCSlot / 2 + a * kAtom, &tm_C, &bs->bc_full[sl], a * 64, g,
                                (int)U.t0, U.b);
                }
                ++m;
                for (int kh = 0; kh < kh_n; ++kh) {
                    const int xs = n % kXStages;
                    if (!wait_bar_idle(&bs->x_empty[xs], ((n / kXStages) & 1) ^ 1, bs, err)) goto pdrain;
                    mbar_arrive_expect_tx(&bs->x_full[xs], kAtom);
                    tma_load_4d(smem + kOffX + xs * kAtom, &tm_x, &bs->x_full[xs], 0,
                                U.hb * kh_n + kh, (int)U.t0, U.b);
                    ++n;
                }
            }
        pdrain:
            // No TMA load may still be writing shared memory when the CTA exits: wait for
            // the last load issued into each slot (already complete unless a role aborted).
            for (int i = 0; i < kXStages && i < n; ++i)
                mbar_wait(&bs->x_full[i], ((n - 1 - i) / kXStages) & 1, 1u << 22);
            for (int i = 0; i < 2 && i < m; ++i) mbar_wait(&bs->bc_full[i], ((m - 1 - i) / 2) & 1, 1u << 22);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idG = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idS = idesc_bf16(128, kP, 1, 1);
            constexpr uint32_t idY = idesc_bf16(128, kP, 0, 1);
            const uint64_t dSB = sw128_desc(smem_u32(smem + kOffWX), kAtom, 1024);
            const uint64_t dRB = sw128_desc(smem_u32(smem + kOffH), kAtom, 1024);
            // G = C B^T of unit m's tile (the diagonal block), shared by the unit's
            // heads; its slot is free once the mask group has used the previous G
            auto issue_g = [&](int m) -> bool {
                const int sl = m & 1;
                if (!MMA_WAIT(&bs->bc_full[sl], (m >> 1) & 1, bs, err)) return false;
                if (!MMA_WAIT(&bs->g_empty, (m & 1) ^ 1, bs, err)) return false;
                tc_fence_after();
                const uint32_t gB = smem_u32(smem + kOffBC + sl * kBCSlot);
                const uint64_t dGA = sw128_desc(gB + kBCSlot / 2, 16, 1024);
                const uint64_t dGB = sw128_desc(gB, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < kN / 16; ++kk) {
                    // start address advances by (kk/4) atoms + (kk%4) x 32 bytes
                    const uint64_t off = (uint64_t)(((kk >> 2) * kAtom + (kk & 3) * 32) >> 4);
                    mma_bf16(tmem + kColG, dGA + off, dGB + off, idG, kk > 0);
                }
                mma_commit(&bs->g_full);
                return true;
            };
            int n = 0, m = 0, pph = 0;
            if (blockIdx.x < prm.nunits && !issue_g(0)) goto drain;
            for (int u = blockIdx.x; u < prm.nunits; u += gridDim.x, ++m) {
                const int sl = m & 1;
                const uint32_t aB = smem_u32(smem + kOffBC + sl * kBCSlot);
                const uint64_t dSA = sw128_desc(aB, kAtom, 1024);
                const uint64_t dRA = sw128_desc(aB + kBCSlot / 2, 16, 1024);
                // one head-independent masked product for the whole unit, or one per head
                if (!MMA_WAIT(&bs->cs_full[n % kCsStages], (n / kCsStages) & 1, bs, err)) goto drain;
                const bool shared =
                    reinterpret_cast<const float*>(smem + kOffCs + (n % kCsStages) * kCsSlot)[6 * kTile + 1] != 0.f;
                for (int kh = 0; kh < kh_n; ++kh, ++n) {
                    const uint32_t pn = n & 1;
                    const int yb = n & 1, xs = n % kXStages;
                    // S += B^T (w o x) onto the preloaded exp(cs_last) h: the head's state
                    // after the tile, which the state group waits on first
                    if (!MMA_WAIT(&bs->wx_full, pn, bs, err)) goto drain;
                    if (!MMA_WAIT(&bs->h_full, pn, bs, err)) goto drain;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk) {
                        const uint64_t rows = (uint64_t)(kk * (2048 >> 4));   // 16 rows of 128 B
                        mma_bf16(tmem + kColS, dSA + rows, dSB + rows, idS, 1u);
                    }
                    if (!shared) mma_commit(&bs->wx_empty);
                    mma_commit(&bs->s_full);
                    // R = C h^T into buffer yb (free once item n-2's epilogue drained it)
                    if (!MMA_WAIT(&bs->ry_empty[yb], ((n >> 1) & 1) ^ 1, bs, err)) goto drain;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kN / 16; ++kk) {
                        const uint64_t rows = (uint64_t)(kk * (2048 >> 4));
                        const uint64_t kofs = (uint64_t)(((kk >> 2) * kAtom + (kk & 3) * 32) >> 4);
                        mma_bf16(tmem + kColR + 64 * yb, dRA + kofs, dRB + rows, idY, kk > 0);
                    }
                    mma_commit(&bs->h_empty);
                    // Y = P x, or Y' = P' (w o x) with the unit's shared P' (P straight from TMEM)
                    if (!shared || kh == 0) {
                        if (!MMA_WAIT(&bs->p_full, pph & 1, bs, err)) goto drain;
                    }
                    if (!shared && !MMA_WAIT(&bs->x_full[xs], (n / kXStages) & 1, bs, err)) goto drain;
                    tc_fence_after();
                    const uint64_t dXB =
                        shared ? dSB : sw128_desc(smem_u32(smem + kOffX + xs * kAtom), kAtom, 1024);
#pragma unroll
                    for (int kk = 0; kk < kTile / 16; ++kk)
                        mma_bf16_tmem_a(tmem + kColY + 64 * yb, tmem + kColP + 8 * kk,
                                        dXB + (uint64_t)(kk * (2048 >> 4)), idY, kk > 0);
                    if (!shared || kh == kh_n - 1) {
                        mma_commit(&bs->p_empty);
                        ++pph;
                    }
                    if (shared) mma_commit(&bs->wx_empty);
                    mma_commit(&bs->x_empty[xs]);
                    mma_commit(&bs->y_full[yb]);
                }
                // every product reading this unit's B/C has been issued
                mma_commit(&bs->bc_empty[sl]);
                if (u + (int)gridDim.x < prm.nunits && !issue_g(m + 1)) goto drain;
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
            const int len = (int)min((int64_t)kTile, T - U.t0);
            // Does every head of the unit decay by at most kSharedMaskRangeLog2 over this
            // tile? Then the unit shares one head-independent masked product.
            float worst = 0.f;
            for (int k2 = 0; k2 < kh_n; ++k2) {
                const int h2 = U.hb * kh_n + k2;
                float sdt = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = lane * 4 + e;
                    sdt += t < len ? __ldg(prm.dt + ((int64_t)U.b * T + U.t0 + t) * H + h2) : 0.f;
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) sdt += __shfl_xor_sync(0xffffffffu, sdt, off);
                worst = fmaxf(worst, sdt * fabsf(prm.A[h2]) * kLog2e);
            }
            const float unit_shared = worst <= kSharedMaskRangeLog2 ? 1.f : 0.f;
            for (int kh = 0; kh < kh_n; ++kh, ++n) {
                const int h = U.hb * kh_n + kh;
                const float a2 = prm.A[h] * kLog2e;
                const float d_h = prm.D ? prm.D[h] : 0.f;
                const int cb = n % kCsStages;
                if (!__all_sync(0xffffffffu, wait_bar_idle(&bs->cs_empty[cb], ((n / kCsStages) & 1) ^ 1, bs, err))) goto done;
                float dtv[4], v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = lane * 4 + e;
                    dtv[e] = t < len ? __ldg(prm.dt + ((int64_t)U.b * T + U.t0 + t) * H + h) : 0.f;
                }
                // The state entering tile t of (b, h) is tile t-1's: wait for its flag here,
                // ahead of the consumers (cs_full, arrived after this acquire, orders the
                // state group's loads of that state after it).
                int bad = 0;
                if (U.t > 0 && lane == 0) {
                    const int* f = prm.flags + (int64_t)U.b * H + h;
                    bool ok = false;
                    const uint64_t t0 = global_ns();
                    for (uint32_t it = 0;; ++it) {
                        if (ld_acquire(f) >= U.t + (prm.stall ? (1 << 30) : 0)) { ok = true; break; }
                        if (it >= 4) __nanosleep(64);
                        if ((it & 15) == 15 &&
                            (*(volatile int*)&bs->abort || global_ns() - t0 > 2000000000ull))
                            break;
                    }
                    if (!ok) {
                        *(volatile int*)&bs->abort = 1;
                        atomicExch(err, 1);
                        bad = 1;
                    }
                }
                if (__any_sync(0xffffffffu, bad)) goto done;
                __syncwarp();
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
                // cs at the last row of this lane's 32-column block (lanes 8b..8b+7 hold block b)
                const float cref = __shfl_sync(0xffffffffu, incl, (lane | 7));
                float4 c4, d4, w4, u4, v4, q4;
                float* cp = &c4.x;
                float* dp = &d4.x;
                float* wp = &w4.x;
                float* up = &u4.x;
                float* vp = &v4.x;
                float* qp = &q4.x;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float ce = excl + v[e];
                    cp[e] = ce;
                    dp[e] = dtv[e];
                    wp[e] = ex2(last - ce) * dtv[e];
                    up[e] = ex2(ce);
                    vp[e] = ex2(cref - ce) * dtv[e];
                    qp[e] = ex2(ce - last);
                }
                reinterpret_cast<float4*>(cs)[lane] = c4;
                reinterpret_cast<float4*>(cs + kTile)[lane] = d4;
                reinterpret_cast<float4*>(cs + 2 * kTile)[lane] = w4;
                reinterpret_cast<float4*>(cs + 3 * kTile)[lane] = u4;
                reinterpret_cast<float4*>(cs + 4 * kTile)[lane] = v4;
                reinterpret_cast<float4*>(cs + 5 * kTile)[lane] = q4;
                if (lane == 0) {
                    cs[6 * kTile] = d_h;
                    cs[6 * kTile + 1] = unit_shared;
                }
                __syncwarp();
                mbar_arrive(&bs->cs_full[cb]);
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
                    const int ps = np % kPubStages;
                    if (!wait_bar_idle(&bs->pub_full[ps], (np / kPubStages) & 1, bs, err)) goto done;
                    __threadfence();
                    st_release(prm.flags + (int64_t)U.b * H + U.hb * kh_n + kh, U.t + 1);
                    mbar_arrive(&bs->pub_empty[ps]);
                }
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ mask group
        // Per unit: when every head's decay over the tile is within range, one
        // head-independent P' = tril(G) (bf16) serves all the unit's heads (their decay
        // goes into w o x and the epilogue); otherwise, per item, P = G o L of the head.
        // Per item: w o x (the S product's operand, and Y's with P').
        const int wq = warp - 4;
        const int j = tid - 128;  // row of the tile == TMEM lane
        const int jj = j & 31;    // row within this warp's diagonal block
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        int n = 0, m = 0, pph = 0;
        for (int u = blockIdx.x; u < prm.nunits; u += gridDim.x, ++m) {
            if (!wait_bar_all(&bs->g_full, m & 1, bs, err)) goto done;
            if (!wait_bar_all(&bs->cs_full[n % kCsStages], (n / kCsStages) & 1, bs, err)) goto done;
            const bool shared =
                reinterpret_cast<const float*>(smem + kOffCs + (n % kCsStages) * kCsSlot)[6 * kTile + 1] != 0.f;
            if (shared) {
                if (!wait_bar_all(&bs->p_empty, (pph & 1) ^ 1, bs, err)) goto done;
                tc_fence_after();
                __syncwarp();
#pragma unroll 1
                for (int blk = 0; blk < 4; ++blk) {
                    uint32_t pk[16];
                    if (blk > wq) {
#pragma unroll
                        for (int q = 0; q < 16; ++q) pk[q] = 0u;
                    } else {
                        float gv[32];
                        tmem_ld32(tmem + lane_base + kColG + 32 * blk, gv);
                        tmem_ld_wait_regs(gv);
                        if (blk < wq) {
#pragma unroll
                            for (int q = 0; q < 16; ++q) pk[q] = pack_bf16(gv[2 * q], gv[2 * q + 1]);
                        } else {
#pragma unroll
                            for (int q = 0; q < 16; ++q)   // causal mask: column i kept while i <= row
                                pk[q] = pack_bf16(2 * q <= jj ? gv[2 * q] : 0.f, 2 * q + 1 <= jj ? gv[2 * q + 1] : 0.f);
                        }
                    }
                    tmem_st16(tmem + lane_base + kColP + 16 * blk, pk);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bs->p_full);
                ++pph;
                mbar_arrive(&bs->g_empty);
            }
            for (int kh = 0; kh < kh_n; ++kh, ++n) {
                const int cb = n % kCsStages;
                if (!wait_bar_all(&bs->cs_full[cb], (n / kCsStages) & 1, bs, err)) goto done;
                const float* cs = reinterpret_cast<const float*>(smem + kOffCs + cb * kCsSlot);
                const float* dts = cs + kTile;
                const float* vv = cs + 4 * kTile;
                // w o x: row j of the x tile scaled by w_j = exp(cs_last - cs_j) dt_j, the
                // B operand of the S product
                {
                    const int xs = n % kXStages;
                    if (!wait_bar_all(&bs->x_full[xs], (n / kXStages) & 1, bs, err)) goto done;
                    if (!wait_bar_all(&bs->wx_empty, (n & 1) ^ 1, bs, err)) goto done;
                    const float w = cs[2 * kTile + j];
                    const float2 w2 = make_float2(w, w);
                    const uint8_t* sx = smem + kOffX + xs * kAtom;
                    uint8_t* swx = smem + kOffWX;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t off = sw128_off(j, c);
                        const uint4 xv = *reinterpret_cast<const uint4*>(sx + off);
                        *reinterpret_cast<uint4*>(swx + off) =
                            make_uint4(pack_bf16(mul2(w2, unpack_bf16(xv.x))), pack_bf16(mul2(w2, unpack_bf16(xv.y))),
                                       pack_bf16(mul2(w2, unpack_bf16(xv.z))), pack_bf16(mul2(w2, unpack_bf16(xv.w))));
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(&bs->wx_full);
                    mbar_arrive(&bs->x_empty[xs]);
                }
                if (shared) {
                    mbar_arrive(&bs->cs_empty[cb]);
                    continue;
                }
                if (!wait_bar_all(&bs->p_empty, (pph & 1) ^ 1, bs, err)) goto done;
                tc_fence_after();
                __syncwarp();
                const float csj = cs[j];
#pragma unroll 1
                for (int blk = 0; blk < 4; ++blk) {
                    uint32_t pk[16];
                    if (blk > wq) {
#pragma unroll
                        for (int q = 0; q < 16; ++q) pk[q] = 0u;
                    } else {
                        float gv[32];
                        tmem_ld32(tmem + lane_base + kColG + 32 * blk, gv);
                        // exp(cs_j - cs_i) dt_i = exp(cs_j - cs_e) * v_i with e the last row of
                        // column block blk and v_i = exp(cs_e - cs_i) dt_i (<= dt_i). Below the
                        // diagonal block the first factor is <= 1 too; on it, it is >= 1 and
                        // bounded by the block's own cs range, which decides whether the
                        // factored form is safe in fp32 or the exponent is taken per element.
                        const float ce = cs[32 * blk + 31];
                        const float a = ex2(csj - ce);
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
                                const float m0 = ex2(csj - c4.x) * d4.x;
                                const float m1 = ex2(csj - c4.y) * d4.y;
                                const float m2 = ex2(csj - c4.z) * d4.z;
                                const float m3 = ex2(csj - c4.w) * d4.w;
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
                ++pph;
                if (kh == kh_n - 1) mbar_arrive(&bs->g_empty);
                mbar_arrive(&bs->cs_empty[cb]);
            }
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ state / epilogue group
        // Iteration n finishes item n and prepares item n+1:
        //   1. the next head's entering state is fetched (its loads in flight),
        //   2. S_n, the state of item n's head after its tile, goes from TMEM onto the chain,
        //   3. the bf16 state operand and exp(cs_last) h preloaded into S, both for item
        //      n+1, so its products run on the tensor pipe during step 4,
        //   4. y_n = Y_n + exp(cs) R_n + D x_n.
        const int q = warp & 3;                 // TMEM lane quarter
        const int ph = (warp - 8) >> 2;         // half of the head dim this warp owns
        const int r = q * 32 + lane;            // tile row for outputs, state index n
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const int64_t PN = (int64_t)kP * kN;
        // Fetching the next unit's state before this item's state is handed on is safe
        // only if that state's predecessors are all earlier units than this one (more
        // units per tile than CTAs); otherwise it waits for the hand-off.
        const bool early_ok = prm.batch * (H / kh_n) > (int)gridDim.x;
        int npub = 0;
        int ystore_xs = -1;   // x slot of this quarter's last y store (issuing lanes)
        float hn[32];    // h[32 ph + i][r] entering the next item's tile
        // the state of head h entering tile U.t (item `item`); returns false on abort.
        // Tile t-1's flag was acquired by the cumsum warp before it released the item's
        // cs slot, so waiting for that slot orders these loads after the flag.
        auto fetch = [&](const Unit& U, int h, int item) -> bool {
            if (!wait_bar_all(&bs->cs_full[item % kCsStages], (item / kCsStages) & 1, bs, err))
                return false;
            if (U.t == 0) {
                const float* src =
                    prm.init ? prm.init + ((int64_t)U.b * H + h) * PN + (int64_t)(32 * ph) * kN + r : nullptr;
#pragma unroll
                for (int i = 0; i < 32; ++i) hn[i] = src ? __ldg(src + (int64_t)i * kN) : 0.f;
                return true;
            }
            const float* src = prm.chain + ((int64_t)U.b * H + h) * PN + (int64_t)(32 * ph) * kN + r;
#pragma unroll
            for (int i = 0; i < 32; ++i) hn[i] = __ldcg(src + (int64_t)i * kN);
            return true;
        };
        // items in the order every role walks them: nx is the next one (unit, head),
        // cur the one being finished
        int nx_u = blockIdx.x, nx_kh = 0;
        bool nx_ok = nx_u < prm.nunits;
        Unit nxU{};
        if (nx_ok) nxU = decode(prm, nx_u);
        bool cur_ok = false;
        int cur_b = 0, cur_h = 0;
        int64_t cur_t0 = 0;
        for (int n = -1; cur_ok || nx_ok; ++n) {
            const int item = n + 1;
            const int nh = nxU.hb * kh_n + nx_kh;   // head of the next item
            // 1. the next item's entering state
            const bool early = nx_ok && (nx_kh != 0 || early_ok);
            if (early && !fetch(nxU, nh, item)) goto done;
            // 2. S_n (this warp's 32 columns) is the state after item n's tile: hand it on
            if (cur_ok) {
                if (!wait_bar_all(&bs->s_full, n & 1, bs, err)) goto done;
                tc_fence_after();
                __syncwarp();
                float sv[32];
                tmem_ld32(tmem + lane_base + kColS + 32 * ph, sv);
                tmem_ld_wait();
                const int ps = npub % kPubStages;
                if (!wait_bar_all(&bs->pub_empty[ps], ((npub / kPubStages) & 1) ^ 1, bs, err))
                    goto done;
                float* dst = prm.chain + ((int64_t)cur_b * H + cur_h) * PN + (int64_t)(32 * ph) * kN + r;
#pragma unroll
                for (int i = 0; i < 32; ++i) __stcg(dst + (int64_t)i * kN, sv[i]);
                mbar_arrive(&bs->pub_full[ps]);
                ++npub;
            }
            if (nx_ok && !early && !fetch(nxU, nh, item)) goto done;
            // 3. operands of the next item
            if (nx_ok) {
                const float* cs1 = reinterpret_cast<const float*>(smem + kOffCs + (item % kCsStages) * kCsSlot);
                // bf16 entering state, the B operand of C h^T (free once R_n is done) ...
                if (!wait_bar_all(&bs->h_empty, (item & 1) ^ 1, bs, err)) goto done;
                write_h_half(smem + kOffH, r, ph, hn);
                fence_proxy_async_smem();
                // ... and exp(cs_last) h preloaded into S (drained in step 2), which the
                // S product then accumulates onto
                {
                    const float e = cs1[4 * kTile - 1];   // exp(cs_last): decay over the tile
                    uint32_t pre[16];
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) pre[i] = __float_as_uint(e * hn[16 * hf + i]);
                        tmem_st16(tmem + lane_base + kColS + 32 * ph + 16 * hf, pre);
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                mbar_arrive(&bs->h_full);
            }
            // 4. y of item n from R and Y (this warp's 32 columns):
            // y_j = Y_j + exp(cs_j) R_j + D x_j, this thread's bytes of row r, written over
            // the same bytes of the item's x tile; each lane quarter's 32 rows then go
            // out as one TMA store
            if (cur_ok) {
                const int yb = n & 1, xs = n % kXStages, cb = n % kCsStages;
                const float* cs = reinterpret_cast<const float*>(smem + kOffCs + cb * kCsSlot);
                if (!wait_bar_all(&bs->y_full[yb], (n >> 1) & 1, bs, err)) goto done;
                tc_fence_after();
                __syncwarp();
                const float uj = cs[3 * kTile + r];
                const float D_h = cs[6 * kTile];
                // shared-mask units produced Y' = tril(C B^T) (w o x): row r scales by
                // exp2(cs_r - cs_last)
                const float qj = cs[6 * kTile + 1] != 0.f ? cs[5 * kTile + r] : 1.f;
                const float2 u2 = make_float2(uj, uj), d2 = make_float2(D_h, D_h), q2 = make_float2(qj, qj);
                uint8_t* sx = smem + kOffX + xs * kAtom;
#pragma unroll 1
                for (int hf = 0; hf < 2; ++hf) {
                    float yv[16], rv[16];
                    tmem_ld16(tmem + lane_base + kColY + 64 * yb + 32 * ph + 16 * hf, yv);
                    tmem_ld16(tmem + lane_base + kColR + 64 * yb + 32 * ph + 16 * hf, rv);
                    uint4 xq[2];
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        xq[c] = *reinterpret_cast<const uint4*>(sx + sw128_off(r, 4 * ph + 2 * hf + c));
                    tmem_ld_wait();
                    if (hf == 1 && ph == 1) {
                        tc_fence_before();
                        mbar_arrive(&bs->ry_empty[yb]);
                    }
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const uint32_t xw[4] = {xq[c].x, xq[c].y, xq[c].z, xq[c].w};
                        uint32_t o[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const int i0 = 8 * c + 2 * e2;
                            const float2 t = fma2(u2, make_float2(rv[i0], rv[i0 + 1]),
                                                  mul2(q2, make_float2(yv[i0], yv[i0 + 1])));
                            o[e2] = pack_bf16(fma2(d2, unpack_bf16(xw[e2]), t));
                        }
                        *reinterpret_cast<uint4*>(sx + sw128_off(r, 4 * ph + 2 * hf + c)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
                // y bytes visible to the async proxy, then the quarter's store: warp 12+q
                // signals (one barrier per item parity), the first lane of warp 8+q issues
                // once both halves are written. Warp 8+q releases R and Y only after that
                // wait, so item n+2's products (and warp 12+q's next arrival on this
                // parity's barrier) cannot come before it.
                fence_proxy_async_smem();
                if (ph == 1) {
                    mbar_arrive(&bs->y_staged[2 * q + (n & 1)]);
                } else {
                    __syncwarp();
                    int ok = 1;
                    if (lane == 0) {
                        ok = wait_bar(&bs->y_staged[2 * q + (n & 1)], (n >> 1) & 1, bs, err);
                        if (ok) {
                            // the previous store from this quarter has read its slot: release it
                            if (ystore_xs >= 0) {
                                bulk_wait_group_read0();
                                mbar_arrive(&bs->x_empty[ystore_xs]);
                                ystore_xs = -1;
                            }
                            if (cur_t0 + 32 * q < T) {   // rows past T are clipped by the store
                                tma_store_4d(&tm_y, sx + q * (kAtom / 4), 0, cur_h, (int)(cur_t0 + 32 * q),
                                             cur_b);
                                bulk_commit_group();
                                ystore_xs = xs;
                            } else {
                                mbar_arrive(&bs->x_empty[xs]);
                            }
                        }
                    }
                    if (!__shfl_sync(0xffffffffu, ok, 0)) goto done;
                    tc_fence_before();
                    mbar_arrive(&bs->ry_empty[yb]);
                }
                mbar_arrive(&bs->cs_empty[cb]);
            }
            // step the item iterator
            cur_ok = nx_ok;
            if (nx_ok) {
                cur_b = nxU.b;
                cur_h = nh;
                cur_t0 = nxU.t0;
                if (++nx_kh >= kh_n) {
                    nx_kh = 0;
                    nx_u += gridDim.x;
                    nx_ok = nx_u < prm.nunits;
                    if (nx_ok) nxU = decode(prm, nx_u);
                }
            }
        }
    }
done:
    // bulk stores still reading shared memory (y tiles) finish before the CTA exits
    if (warp >= 8 && warp < 12 && lane == 0) bulk_wait_group0();
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
    prm.H = (int)d.H;
    prm.G = (int)d.G;
    prm.kheads = kheads;
    prm.batch = (int)d.b;
    const int64_t ntiles = (d.T + kTile - 1) / kTile;
    const int64_t nunits = ntiles * d.b * (d.H / kheads);
    if (nunits > INT32_MAX || d.T > INT32_MAX) return cudaErrorInvalidValue;
    prm.nunits = (int)nunits;
    // SSD_TEST_STALL_CHAIN=1 makes every chain hand-off wait run out (about 2 s), so
    // that tests can check the device status path without faulting the GPU
    const char* stall = getenv("SSD_TEST_STALL_CHAIN");
    prm.stall = (stall && stall[0] == '1') ? 1 : 0;
    e = cudaFuncSetAttribute(ssd_fused_ws_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const int grid = prm.nunits < g_num_sms ? prm.nunits : g_num_sms;
    ssd_fused_ws_kernel<<<grid, kThreads, kSmemBytes, st>>>(maps[0], maps[1], maps[2], maps[3], prm);
    return cudaGetLastError();
}

}  // namespace ssd
