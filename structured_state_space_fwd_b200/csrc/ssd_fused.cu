// Warp-specialized, persistent single-pass SSD forward for sm_100a.
//
// "Transformers are SSMs" (Knowl 1, 2, 3, 7) with the chunk equal to one
// 128-token tile: per tile the diagonal block in the quadratic masked form,
// everything before the tile through the state entering it. With cs the
// inclusive cumulative sum of dt*A inside the tile (log2 units), L = cs of the
// tile's last token, w_i = 2^(L - cs_i) dt_i and q_j = 2^(cs_j - L), the
// tile's outputs and leaving state are
//
//   y_j  = q_j [ (tril(C B^T) (w o x))_j + C_j . (2^L h) + D x_j / q_j ]
//   h'   = 2^L h + B^T (w o x)
//
// (the 1-semiseparable mask of Knowl 3 factored through the tile's last token).
// The three terms in brackets accumulate in ONE tensor-memory accumulator Y'':
// the skip term is stored into it first, then the masked product and the
// state term are added by the tensor cores, so the epilogue is one scaling.
// The tile-local products S = B^T (w o x) and tril(C B^T)(w o x) do not depend
// on the state entering the tile; only the element-wise h' = 2^L h + S and
// the product C (2^L h)^T wait for it. A unit whose heads decay by more than
// 2^96 over the tile takes the unfactored form instead: per head
// P = (C B^T) o exp(segsum) o dt (exponent per element), Y = P x + D x, and
// R = C h^T into a separate accumulator, y = Y + 2^cs R.
//
// Roles (16 warps):
//   warp 0      TMA producer; takes units from a global ticket and hands their
//               ids to every role through a small ring
//   warp 1      TMEM owner and MMA issuer (one thread)
//   warp 2      per item: dt loads, cumulative sum, the chain flag of the
//               state entering the tile (acquire)
//   warp 3      chain publisher: releases the flag of each head's leaving state
//   warps 4-7   mask group (thread = token row): tril(C B^T) into TMEM once per
//               unit, per item the skip-term preload and w o x in place
//   warps 8-11  chain group (thread = state row): per item the leaving state
//               onto the chain and the bf16 state operand of C h^T
//   warps 12-15 epilogue group (thread = token row): per item y = q Y'' staged
//               in shared memory, one TMA store per warp
// The chain and epilogue groups run their own loops: a head's state update does
// not wait for the previous item's output, only for the operand buffer it reuses
// (two buffers, each also the staging of one item's y).
//
// Work: a unit is (tile t, batch row b, block of k heads of one group), units
// in tile-major order, handed out by an atomic ticket so that a unit's
// predecessor on its chain (same b and heads, tile t-1) was always taken
// earlier by a CTA that is running. An item is (unit, head). The state of
// (b, h) after tile t goes to tile t+1 through one L2-resident buffer and a
// release/acquire flag. Optionally the sequence is cut into segments of
// `seg_tiles` tiles whose entering states were computed beforehand (segment
// states and a scan over them, ssd_segment.cu); then each segment is a chain
// of its own and many short chains run side by side.
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
constexpr int kThreads = 640;
constexpr int kCsSlots = 2;
constexpr int kYSlots = 3;
constexpr int kURing = 4;
constexpr int kPubStages = 4;

constexpr uint32_t kAtom = kTile * 128;    // 16 KB: 128 rows of 128 bytes (64 bf16)
// per item: cs[128], dt[128], then L (cs of the last token), D_h, unit mode
constexpr uint32_t kCsSlotBytes = 2 * kTile * 4 + 64;
constexpr int kCsL = 2 * kTile, kCsD = 2 * kTile + 1, kCsMode = 2 * kTile + 2;

// TMEM columns: G = C B^T (fp32), P (bf16 pairs, the A operand of the masked
// product), S slots, three Y'' accumulators
constexpr uint32_t kColG = 0;
constexpr uint32_t kColP = 128;
constexpr uint32_t kColS = 192;
constexpr uint32_t kColY = 320;

constexpr float kLog2e = 1.4426950408889634f;
// Widest decay over one tile (log2 units) for which a unit takes the factored
// form: 2^(L - cs) dt (bf16 operand) and 2^(L - cs) (skip-term divisor) then stay
// inside the normal fp32 / bf16 exponent range with a wide margin.
constexpr float kSharedMaskRangeLog2 = 96.f;

// Shared-memory layout for state capacity NS (128 or 256 state elements).
// per Y'' accumulator: the epilogue's row factor (q_j, or 2^cs_j), then 2^L, unit mode
constexpr uint32_t kYInfoBytes = kTile * 4 + 16;

// B and C tiles live in a ring of tile buffers, taken in the order B_0, C_0, B_1,
// C_1, ...: a unit's B is released once its S products are done, its C once its
// state products are, so three buffers let the next unit's tiles load early.
template <int NS>
struct Cfg {
    static constexpr int kAtoms = NS / 64;                  // 64-wide column atoms of B or C
    static constexpr uint32_t kBCTile = kAtoms * kAtom;     // B (or C) tile of one unit
    static constexpr int kBufs = NS == 128 ? 3 : 2;         // tile buffers
    static constexpr int kXSlots = NS == 128 ? 4 : 3;
    static constexpr int kSSlots = NS == 128 ? 2 : 1;
    static constexpr int kMHalves = NS / 128;               // 128-row halves of the state
    static constexpr int kHYSlots = NS == 128 ? 2 : 1;      // state operand buffers
    static constexpr uint32_t kHYBytes = NS * 128;          // NS rows of 64 bf16
    // y staging: its own 4 KB per epilogue warp, or (NS = 256) the operand buffer
    static constexpr bool kOwnStaging = NS == 128;
    static constexpr uint32_t kOffBC = 0;
    static constexpr uint32_t kOffX = kOffBC + kBufs * kBCTile;
    static constexpr uint32_t kOffHY = kOffX + kXSlots * kAtom;
    static constexpr uint32_t kOffStage = kOffHY + kHYSlots * kHYBytes;
    static constexpr uint32_t kOffCs = kOffStage + (kOwnStaging ? kAtom : 0);
    static constexpr uint32_t kOffYInfo = kOffCs + kCsSlots * kCsSlotBytes;
    static constexpr uint32_t kOffBar = kOffYInfo + kYSlots * kYInfoBytes;
    static constexpr uint32_t kSmem = kOffBar + 1024;
    static_assert(kSmem <= 232448, "shared memory budget");
    static_assert(kColY + kYSlots * 64 <= 512, "tensor memory budget");
};

struct Params {
    const float* dt;
    const float* A;
    const float* D;
    const float* init;    // [b,H,P,N] or null (zeros)
    float* finalbuf;      // chain buffer of the last segment: final states or workspace
    float* segbuf;        // [b,nseg,H,P,N]: slot s >= 1 holds the state entering segment s
    int* ticket;
    int* error;
    int* flags;           // [b*nseg*H] tiles of the segment whose leaving state is out
    int64_t T;
    int H, G, N, kheads, batch, nunits, ntiles, seg_tiles, nseg;
    int stall;            // test builds only: chain flags awaited at a value never reached
};

struct Bars {
    uint64_t u_full[kURing], u_empty[kURing];
    uint64_t tb_full[3], tb_empty[3];
    uint64_t x_full[4], x_empty[4];
    uint64_t wx_full[4];          // item's operands ready (w o x, or P and raw x); mode in xmode
    uint64_t wx2_full;            // unfactored item: x scaled in place after Y = P x
    uint64_t g_full, g_empty, p_full, p_empty, xr_done;
    uint64_t cs_full[kCsSlots], cs_empty[kCsSlots];
    uint64_t s_full[2], s_empty[2];
    uint64_t y_full[kYSlots], y_empty[kYSlots], yi_full[kYSlots];
    uint64_t h_full[2], hy_free[2];
    uint64_t pub_full[kPubStages], pub_empty[kPubStages];
    uint64_t fin;
    int uid[kURing];
    int xmode[4];
    uint32_t tmem;
    int abort;
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

// arrivals on u_empty: MMA thread, cumsum warp, publisher, mask, chain and epilogue groups
constexpr uint32_t kUnitReaders = 1 + 32 + 1 + 128 + 256 + 128;

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
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// 2^x on the special-function unit (a few ulp; results below 2^-126 flush to
// zero, i.e. decays too small to matter).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // every wait gives up after about 2 s

// Bounded mbarrier wait that also gives up once another role aborted (checked
// every 16 polls). The polling loop is out of line: one copy in the
// instruction caches for every call site.
__device__ __noinline__ bool wait_bar_slow(uint64_t* bar, uint32_t parity, Bars* bs, int* err,
                                           uint32_t sleep_ns) {
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (sleep_ns) __nanosleep(sleep_ns);
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 15) == 0) {
            if (*(volatile int*)&bs->abort) return false;
            if (global_ns() - t0 > kWaitLimitNs) {
                *(volatile int*)&bs->abort = 1;
                atomicExch(err, 3);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Bars* bs, int* err) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bar_slow(bar, parity, bs, err, 0);
}
// For roles that run ahead of their consumers (producer, cumsum warp, publisher):
// sleeping between polls leaves the issue slots to the compute warps.
__device__ __forceinline__ bool wait_bar_idle(uint64_t* bar, uint32_t parity, Bars* bs, int* err) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bar_slow(bar, parity, bs, err, 100);
}
// Called by all 32 lanes of a warp together (the compute groups): the outcome is
// warp-uniform, so no lane leaves a loop its warp-mates stay in (tcgen05.ld/st are
// warp-collective). A waiting warp is suspended by the barrier (time-limited hint)
// rather than spinning, so it leaves the issue slots of its scheduler to the MMA
// thread that shares it.
#ifndef SSD_SUSPEND_NS
#define SSD_SUSPEND_NS 2000u
#endif
__device__ __noinline__ bool wait_bar_sleep_slow(uint64_t* bar, uint32_t parity, Bars* bs, int* err) {
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait_hint(bar, parity, SSD_SUSPEND_NS)) return true;
        if ((i & 3) == 0) {
            if (*(volatile int*)&bs->abort) return false;
            if (global_ns() - t0 > kWaitLimitNs) {
                *(volatile int*)&bs->abort = 1;
                atomicExch(err, 3);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool wait_bar_all(uint64_t* bar, uint32_t parity, Bars* bs, int* err) {
    const bool ok = mbar_try_wait(bar, parity) || wait_bar_sleep_slow(bar, parity, bs, err);
    return __all_sync(0xffffffffu, ok);
}

struct Unit {
    int t, kk, s, b, hb;   // tile, tile within its segment, segment, batch row, head block
    int64_t t0;            // first token of the tile
};
__device__ __forceinline__ Unit decode(const Params& p, int u) {
    const int nhb = p.H / p.kheads;
    Unit r;
    r.hb = u % nhb;
    int q = u / nhb;
    r.b = q % p.batch;
    q /= p.batch;
    r.s = q % p.nseg;
    r.kk = q / p.nseg;
    r.t = r.s * p.seg_tiles + r.kk;
    r.t0 = (int64_t)r.t * kTile;
    return r;
}
__device__ __forceinline__ int64_t chain_index(const Params& p, const Unit& U, int h) {
    return ((int64_t)U.b * p.nseg + U.s) * p.H + h;
}
// buffer that carries (b, h)'s state from tile to tile inside segment s
__device__ __forceinline__ float* chain_buf(const Params& p, const Unit& U, int h) {
    const int64_t PN = (int64_t)kP * p.N;
    if (U.s == p.nseg - 1) return p.finalbuf + ((int64_t)U.b * p.H + h) * PN;
    return p.segbuf + chain_index(p, U, h) * PN;
}
// state entering the unit's tile for head h (null: zeros)
__device__ __forceinline__ const float* entry_src(const Params& p, const Unit& U, int h) {
    const int64_t PN = (int64_t)kP * p.N;
    if (U.kk != 0) return chain_buf(p, U, h);
    if (U.s == 0) return p.init ? p.init + ((int64_t)U.b * p.H + h) * PN : nullptr;
    return p.segbuf + chain_index(p, U, h) * PN;
}

// Byte offset of row `row`, 16-byte chunk `c` in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t c) { return sw128_off(row, c); }

// KS steps of K = 16 over the state dim into D: A K-major (C), B either K-major (B,
// the product G) or N-contiguous rows of 128 bytes (the state operand). Unrolled,
// so consecutive MMAs issue back to back.
template <int KS, bool kBRows>
__device__ __forceinline__ void mma_state_dim(uint32_t d, uint64_t dA, uint64_t dB, uint32_t idesc,
                                              uint32_t acc0) {
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
        const uint64_t kofs = (uint64_t)(((kk >> 2) * kAtom + (kk & 3) * 32) >> 4);
        mma_bf16(d, dA + kofs, dB + (kBRows ? (uint64_t)(kk * (2048 >> 4)) : kofs), idesc, kk > 0 ? 1u : acc0);
    }
}
template <bool kBRows>
__device__ __forceinline__ void mma_state_dim_n(int ks, uint32_t d, uint64_t dA, uint64_t dB, uint32_t idesc,
                                                uint32_t acc0) {
    switch (ks) {
        case 1: mma_state_dim<1, kBRows>(d, dA, dB, idesc, acc0); break;
        case 2: mma_state_dim<2, kBRows>(d, dA, dB, idesc, acc0); break;
        case 4: mma_state_dim<4, kBRows>(d, dA, dB, idesc, acc0); break;
        case 8: mma_state_dim<8, kBRows>(d, dA, dB, idesc, acc0); break;
        default: mma_state_dim<16, kBRows>(d, dA, dB, idesc, acc0); break;
    }
}

template <int NS>
__global__ void __launch_bounds__(kThreads, 1)
    ssd_fused_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_B,
                     const __grid_constant__ CUtensorMap tm_C, const __grid_constant__ CUtensorMap tm_y,
                     const Params prm) {
    using K = Cfg<NS>;
    extern __shared__ __align__(1024) uint8_t smem[];
    Bars* bs = reinterpret_cast<Bars*>(smem + K::kOffBar);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int* err = prm.error;

    if (tid == 0) {
        if ((smem_u32(smem) & 1023u) != 0) atomicExch(err, 4);
        for (int i = 0; i < kURing; ++i) {
            mbar_init(&bs->u_full[i], 1);
            mbar_init(&bs->u_empty[i], kUnitReaders);
        }
        for (int i = 0; i < 3; ++i) {
            mbar_init(&bs->tb_full[i], 1);
            mbar_init(&bs->tb_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bs->s_full[i], 1);
            mbar_init(&bs->s_empty[i], 256);
        }
        for (int i = 0; i < 4; ++i) {
            mbar_init(&bs->x_full[i], 1);
            mbar_init(&bs->x_empty[i], 1);
            mbar_init(&bs->wx_full[i], 128);
        }
        mbar_init(&bs->wx2_full, 128);
        mbar_init(&bs->g_full, 1);
        mbar_init(&bs->g_empty, 128);
        mbar_init(&bs->p_full, 128);
        mbar_init(&bs->p_empty, 1);
        mbar_init(&bs->xr_done, 1);
        for (int i = 0; i < kCsSlots; ++i) {
            mbar_init(&bs->cs_full[i], 32);
            mbar_init(&bs->cs_empty[i], 128);
        }
        for (int i = 0; i < kYSlots; ++i) {
            mbar_init(&bs->y_full[i], 1);
            mbar_init(&bs->y_empty[i], 128);
            mbar_init(&bs->yi_full[i], 128);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bs->h_full[i], 256);
            // freed by the state product's commit, or by the epilogue warps' y stores
            mbar_init(&bs->hy_free[i], K::kOwnStaging ? 1 : 4);
        }
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
    const int kh = prm.kheads;
    const int64_t T = prm.T;
    const int H = prm.H;
    // K steps of the products over the state dim: a power of two covering N (the B
    // and C tiles are loaded whole, zero beyond N, so the extra steps add nothing)
    const int ksN = prm.N <= 16 ? 1 : prm.N <= 32 ? 2 : prm.N <= 64 ? 4 : prm.N <= 128 ? 8 : 16;
    const int natoms = (ksN * 16 + 63) / 64;   // B/C column atoms loaded
    const float* cs_base = reinterpret_cast<const float*>(smem + K::kOffCs);

    if (misaligned) {
        // nothing
    } else if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int m = 0, n = 0, mb = 0;    // units taken, x tiles and tile buffers loaded
            for (;; ++m) {
                int u;
                do {
                    u = atomicAdd(prm.ticket, 1);
                } while (u < prm.nunits && decode(prm, u).t >= prm.ntiles);
                if (u >= prm.nunits) u = -1;
                const int ur = m % kURing;
                if (!wait_bar_idle(&bs->u_empty[ur], ((m / kURing) & 1) ^ 1, bs, err)) goto pdrain;
                bs->uid[ur] = u;
                mbar_arrive(&bs->u_full[ur]);
                if (u < 0) break;
                const Unit U = decode(prm, u);
                const int g = U.hb * kh / (H / prm.G);
                for (int bc = 0; bc < 2; ++bc, ++mb) {    // B, then C
                    const int tb = mb % K::kBufs;
                    if (!wait_bar_idle(&bs->tb_empty[tb], ((mb / K::kBufs) & 1) ^ 1, bs, err)) goto pdrain;
                    mbar_arrive_expect_tx(&bs->tb_full[tb], natoms * kAtom);
                    for (int a = 0; a < natoms; ++a)
                        tma_load_4d(smem + K::kOffBC + tb * K::kBCTile + a * kAtom, bc ? &tm_C : &tm_B,
                                    &bs->tb_full[tb], a * 64, g, (int)U.t0, U.b);
                }
                for (int k = 0; k < kh; ++k, ++n) {
                    const int xs = n % K::kXSlots;
                    if (!wait_bar_idle(&bs->x_empty[xs], ((n / K::kXSlots) & 1) ^ 1, bs, err)) goto pdrain;
                    mbar_arrive_expect_tx(&bs->x_full[xs], kAtom);
                    tma_load_4d(smem + K::kOffX + xs * kAtom, &tm_x, &bs->x_full[xs], 0, U.hb * kh + k,
                                (int)U.t0, U.b);
                }
            }
        pdrain:
            // No TMA load may still be writing shared memory when the CTA exits: wait for
            // the last load issued into each slot (already complete unless a role aborted).
            for (int i = 0; i < K::kXSlots && i < n; ++i)
                mbar_wait(&bs->x_full[(n - 1 - i) % K::kXSlots], ((n - 1 - i) / K::kXSlots) & 1, 1u << 22);
            for (int i = 0; i < K::kBufs && i < mb; ++i)
                mbar_wait(&bs->tb_full[(mb - 1 - i) % K::kBufs], ((mb - 1 - i) / K::kBufs) & 1, 1u << 22);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Per item i: S_i and the masked product (neither waits for the chain), then
        // the previous item's state product C h^T, whose operand the chain group
        // writes once that head's entering state is known.
        if (lane == 0) {
            constexpr uint32_t idG = idesc_bf16(128, 128, 0, 0);   // C (K-major) x B (K-major)
            constexpr uint32_t idS = idesc_bf16(128, kP, 1, 1);    // B^T (N-contiguous) x (w o x)
            constexpr uint32_t idY = idesc_bf16(128, kP, 0, 1);    // P or C (K-major) x (w o x) or h
            struct Pend {
                int item, ys, ss, cb;   // cb: tile buffer of the unit's C
                bool shared, last;
            };
            Pend pv{};
            bool have = false;
            int psh = 0, nsh = 0;
            // C (2^L h)^T onto Y'' (factored units) or C h^T into the item's S slot
            auto issue_r = [&](const Pend& q) -> bool {
                const int hs = q.item % K::kHYSlots;
                if (!wait_bar(&bs->h_full[hs], (q.item / K::kHYSlots) & 1, bs, err)) return false;
                tc_fence_after();
                const uint64_t dH = sw128_desc(smem_u32(smem + K::kOffHY + hs * K::kHYBytes), kAtom, 1024);
                const uint32_t cB = smem_u32(smem + K::kOffBC + q.cb * K::kBCTile);
                const uint64_t dC = sw128_desc(cB, 16, 1024);
                const uint32_t d = q.shared ? tmem + kColY + 64 * q.ys : tmem + kColS + 64 * q.ss;
                mma_state_dim_n<true>(ksN, d, dC, dH, idY, q.shared ? 1u : 0u);
                mma_commit(&bs->y_full[q.ys]);
                if (K::kOwnStaging) mma_commit(&bs->hy_free[hs]);
                if (q.last) mma_commit(&bs->tb_empty[q.cb]);
                return true;
            };
            int m = 0, i = 0;
            for (;; ++m) {
                const int ur = m % kURing;
                if (!wait_bar(&bs->u_full[ur], (m / kURing) & 1, bs, err)) goto drain;
                const int u = bs->uid[ur];
                mbar_arrive(&bs->u_empty[ur]);
                if (u < 0) break;
                const int tbB = (2 * m) % K::kBufs, tbC = (2 * m + 1) % K::kBufs;
                const uint32_t bcB = smem_u32(smem + K::kOffBC + tbB * K::kBCTile);
                const uint32_t bcC = smem_u32(smem + K::kOffBC + tbC * K::kBCTile);
                // G = C B^T of the tile, shared by the unit's heads
                if (!wait_bar(&bs->tb_full[tbB], ((2 * m) / K::kBufs) & 1, bs, err)) goto drain;
                if (!wait_bar(&bs->tb_full[tbC], ((2 * m + 1) / K::kBufs) & 1, bs, err)) goto drain;
                if (!wait_bar(&bs->g_empty, (m & 1) ^ 1, bs, err)) goto drain;
                tc_fence_after();
                {
                    mma_state_dim_n<false>(ksN, tmem + kColG, sw128_desc(bcC, 16, 1024), sw128_desc(bcB, 16, 1024),
                                           idG, 0u);
                }
                mma_commit(&bs->g_full);
                const uint64_t dSA = sw128_desc(bcB, kAtom, 1024);
                for (int k = 0; k < kh; ++k, ++i) {
                    const int xs = i % K::kXSlots, ys = i % kYSlots, ss = i % K::kSSlots;
                    if (!wait_bar(&bs->wx_full[xs], (i / K::kXSlots) & 1, bs, err)) goto drain;
                    const bool shared = *(volatile int*)&bs->xmode[xs] != 0;
                    // a pending unfactored item's C h^T goes into its S slot before this
                    // item's S may reuse that slot
                    if (have && !pv.shared) {
                        if (!issue_r(pv)) goto drain;
                        have = false;
                    }
                    const uint64_t dX = sw128_desc(smem_u32(smem + K::kOffX + xs * kAtom), kAtom, 1024);
                    auto issue_s = [&]() -> bool {
                        if (!wait_bar(&bs->s_empty[ss], ((i / K::kSSlots) & 1) ^ 1, bs, err)) return false;
                        tc_fence_after();
                        for (int mh = 0; mh < K::kMHalves; ++mh)
                            for (int kk = 0; kk < kTile / 16; ++kk)
                                mma_bf16(tmem + kColS + 64 * ss + 64 * mh,
                                         dSA + (uint64_t)((2 * mh * kAtom) >> 4) + (uint64_t)(kk * 128),
                                         dX + (uint64_t)(kk * 128), idS, kk > 0);
                        mma_commit(&bs->s_full[ss]);
                        return true;
                    };
                    if (shared) {
                        tc_fence_after();
                        if (!issue_s()) goto drain;
                        if (k == 0) {
                            if (!wait_bar(&bs->p_full, psh & 1, bs, err)) goto drain;
                            ++psh;
                            tc_fence_after();
                        }
                        for (int kk = 0; kk < kTile / 16; ++kk)
                            mma_bf16_tmem_a(tmem + kColY + 64 * ys, tmem + kColP + 8 * kk,
                                            dX + (uint64_t)(kk * 128), idY, 1u);
                        mma_commit(&bs->x_empty[xs]);
                        if (k == kh - 1) mma_commit(&bs->p_empty);
                    } else {
                        // Y = P x with the raw tile, then S once the tile is scaled in place
                        tc_fence_after();
                        for (int kk = 0; kk < kTile / 16; ++kk)
                            mma_bf16_tmem_a(tmem + kColY + 64 * ys, tmem + kColP + 8 * kk,
                                            dX + (uint64_t)(kk * 128), idY, 1u);
                        mma_commit(&bs->xr_done);
                        mma_commit(&bs->p_empty);
                        if (!wait_bar(&bs->wx2_full, nsh & 1, bs, err)) goto drain;
                        ++nsh;
                        if (!issue_s()) goto drain;
                        mma_commit(&bs->x_empty[xs]);
                    }
                    if (have) {
                        if (!issue_r(pv)) goto drain;
                        have = false;
                    }
                    // the unit's B has served its last S product
                    if (k == kh - 1) mma_commit(&bs->tb_empty[tbB]);
                    pv = Pend{i, ys, ss, tbC, shared, k == kh - 1};
                    have = true;
                    // with two tile buffers the next unit's C reuses this unit's: its last
                    // state product goes out first
                    if (K::kBufs == 2 && k == kh - 1) {
                        if (!issue_r(pv)) goto drain;
                        have = false;
                    }
                }
            }
            if (have && !issue_r(pv)) goto drain;
        drain:
            // every MMA issued so far is complete before TMEM is released
            mma_commit(&bs->fin);
            mbar_wait(&bs->fin, 0, 1u << 24);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ cumsum warp
        // Per unit, the dt of all its heads is loaded at once, and lane k polls head
        // k's chain flag, so no item waits a full memory round trip of its own.
        constexpr int kMaxKh = NS == 256 ? 8 : 4;
        float dtv[kMaxKh][4];
        auto load_dt = [&](const Unit& U, float (&v)[kMaxKh][4]) {
            const int len = (int)min((int64_t)kTile, T - U.t0);
#pragma unroll
            for (int k = 0; k < kMaxKh; ++k)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = lane * 4 + e;
                    v[k][e] = (k < kh && t < len)
                                  ? __ldg(prm.dt + ((int64_t)U.b * T + U.t0 + t) * H + U.hb * kh + k)
                                  : 0.f;
                }
        };
        int m = 0, i = 0;
        for (;; ++m) {
            const int ur = m % kURing;
            if (!__all_sync(0xffffffffu, wait_bar_idle(&bs->u_full[ur], (m / kURing) & 1, bs, err)))
                goto done;
            const int u = bs->uid[ur];
            mbar_arrive(&bs->u_empty[ur]);
            if (u < 0) break;
            const Unit U = decode(prm, u);
            load_dt(U, dtv);
            // Does every head of the unit decay by at most kSharedMaskRangeLog2 over this
            // tile? Then the unit takes the factored form.
            float worst = 0.f;
#pragma unroll
            for (int k = 0; k < kMaxKh; ++k) {
                if (k >= kh) break;
                float sdt = dtv[k][0] + dtv[k][1] + dtv[k][2] + dtv[k][3];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) sdt += __shfl_xor_sync(0xffffffffu, sdt, off);
                worst = fmaxf(worst, sdt * fabsf(__ldg(prm.A + U.hb * kh + k)) * kLog2e);
            }
            const float mode = worst <= kSharedMaskRangeLog2 ? 1.f : 0.f;
            // lane k < kh watches the chain flag of head k (the state entering this tile
            // comes from the previous tile of the same segment)
            const bool watch = U.kk > 0 && lane < kh;
            const int* myflag = prm.flags + chain_index(prm, U, U.hb * kh + (lane < kh ? lane : 0));
            const int want = U.kk + (prm.stall ? (1 << 30) : 0);
            bool seen = !watch;
            const uint64_t tw = global_ns();
#pragma unroll
            for (int k = 0; k < kMaxKh; ++k) {
                if (k >= kh) break;
                const int h = U.hb * kh + k;
                const float a2 = __ldg(prm.A + h) * kLog2e;
                const float d_h = prm.D ? __ldg(prm.D + h) : 0.f;
                const int c = i % kCsSlots;
                if (!__all_sync(0xffffffffu,
                                wait_bar_idle(&bs->cs_empty[c], ((i / kCsSlots) & 1) ^ 1, bs, err)))
                    goto done;
                // acquire head k's flag before the consumers may read its state
                for (uint32_t it = 0;; ++it) {
                    if (!seen) seen = ld_acquire(myflag) >= want;
                    if (__shfl_sync(0xffffffffu, seen ? 1 : 0, k)) break;
                    int bad = 0;
                    if ((it & 15) == 15) {
                        bad = *(volatile int*)&bs->abort ? 2 : (global_ns() - tw > kWaitLimitNs ? 1 : 0);
                        bad = __shfl_sync(0xffffffffu, bad, 0);
                    }
                    if (bad) {
                        if (bad == 1 && lane == 0) {
                            *(volatile int*)&bs->abort = 1;
                            atomicExch(err, 1);
                        }
                        goto done;
                    }
                    if (it >= 2) __nanosleep(64);
                }
                float run = 0.f, v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    run += dtv[k][e] * a2;
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
                float* cs = reinterpret_cast<float*>(smem + K::kOffCs + c * kCsSlotBytes);
                reinterpret_cast<float4*>(cs)[lane] =
                    make_float4(excl + v[0], excl + v[1], excl + v[2], excl + v[3]);
                reinterpret_cast<float4*>(cs + kTile)[lane] =
                    make_float4(dtv[k][0], dtv[k][1], dtv[k][2], dtv[k][3]);
                if (lane == 0) {
                    cs[kCsL] = last;
                    cs[kCsD] = d_h;
                    cs[kCsMode] = mode;
                }
                __syncwarp();
                mbar_arrive(&bs->cs_full[c]);
                ++i;
            }
        }
    } else if (warp == 3) {
        // ------------------------------------------------------------ chain publisher
        // The state group stores a head's leaving state and arrives on pub_full; this lane
        // then makes those stores visible GPU-wide (one fence, cumulative over the stores
        // ordered before the barrier) and releases the chain flag.
        if (lane == 0) {
            int m = 0, np = 0;
            for (;; ++m) {
                const int ur = m % kURing;
                if (!wait_bar_idle(&bs->u_full[ur], (m / kURing) & 1, bs, err)) goto done;
                const int u = bs->uid[ur];
                mbar_arrive(&bs->u_empty[ur]);
                if (u < 0) break;
                const Unit U = decode(prm, u);
                for (int k = 0; k < kh; ++k, ++np) {
                    const int ps = np % kPubStages;
                    if (!wait_bar_idle(&bs->pub_full[ps], (np / kPubStages) & 1, bs, err)) goto done;
                    __threadfence();
                    st_release(prm.flags + chain_index(prm, U, U.hb * kh + k), U.kk + 1);
                    mbar_arrive(&bs->pub_empty[ps]);
                }
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ mask group
        // Thread j owns token row j of the tile (its TMEM lane). Per unit: the masked
        // product's A operand, tril(G) for a factored unit. Per item: the skip term
        // D x_j / q_j (or D x_j) stored into the item's Y'' accumulator, and w o x in
        // place of the x tile (the B operand of S and of the factored masked product).
        // An unfactored item first gets its own P = G o exp(cs_j - cs_i) dt_i and is
        // multiplied with the raw x tile before x is scaled in place.
        const int wq = warp - 4;
        const int j = tid - 128;
        const int jj = j & 31;
        const uint32_t lb = (uint32_t)(wq * 32) << 16;
        int m = 0, i = 0, pph = 0, nsh = 0;
        for (;; ++m) {
            const int ur = m % kURing;
            if (!wait_bar_all(&bs->u_full[ur], (m / kURing) & 1, bs, err)) goto done;
            const int u = bs->uid[ur];
            mbar_arrive(&bs->u_empty[ur]);
            if (u < 0) break;
            if (!wait_bar_all(&bs->cs_full[i % kCsSlots], (i / kCsSlots) & 1, bs, err)) goto done;
            const bool shared = cs_base[(i % kCsSlots) * (kCsSlotBytes / 4) + kCsMode] != 0.f;
            if (!wait_bar_all(&bs->g_full, m & 1, bs, err)) goto done;
            if (shared) {
                if (!wait_bar_all(&bs->p_empty, (pph & 1) ^ 1, bs, err)) goto done;
                tc_fence_after();
                __syncwarp();
#pragma unroll 1
                for (int blk = 0; blk < 4; ++blk) {
                    uint32_t pk[16];
                    if (blk > wq) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = 0u;
                    } else {
                        float gv[32];
                        tmem_ld32(tmem + lb + kColG + 32 * blk, gv);
                        tmem_ld_wait_regs(gv);
                        if (blk < wq) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(gv[2 * e], gv[2 * e + 1]);
                        } else {
#pragma unroll
                            for (int e = 0; e < 16; ++e)   // causal mask: column i kept while i <= row
                                pk[e] = pack_bf16(2 * e <= jj ? gv[2 * e] : 0.f,
                                                  2 * e + 1 <= jj ? gv[2 * e + 1] : 0.f);
                        }
                    }
                    tmem_st16(tmem + lb + kColP + 16 * blk, pk);
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&bs->p_full);
                ++pph;
                mbar_arrive(&bs->g_empty);
            } else {
                tc_fence_after();
            }
            for (int k = 0; k < kh; ++k, ++i) {
                const int c = i % kCsSlots, xs = i % K::kXSlots, ys = i % kYSlots;
                if (!wait_bar_all(&bs->cs_full[c], (i / kCsSlots) & 1, bs, err)) goto done;
                if (!wait_bar_all(&bs->x_full[xs], (i / K::kXSlots) & 1, bs, err)) goto done;
                if (!wait_bar_all(&bs->y_empty[ys], ((i / kYSlots) & 1) ^ 1, bs, err)) goto done;
                const float* cs = cs_base + c * (kCsSlotBytes / 4);
                const float L = cs[kCsL], csj = cs[j];
                const float up = ex2(L - csj);                  // 2^(L - cs_j) <= 1
                const float w = up * cs[kTile + j];             // w_j = 2^(L - cs_j) dt_j
                const float dq = cs[kCsD] * (shared ? up : 1.f);  // D / q_j, or D
                // what the chain and epilogue groups need of this item, kept with its Y''
                {
                    float* yi = reinterpret_cast<float*>(smem + K::kOffYInfo + ys * kYInfoBytes);
                    yi[j] = shared ? ex2(csj - L) : ex2(csj);   // q_j, or 2^cs_j
                    if (j == 0) {
                        yi[kTile] = ex2(L);
                        yi[kTile + 1] = shared ? 1.f : 0.f;
                    }
                    mbar_arrive(&bs->yi_full[ys]);
                }
                uint8_t* sx = smem + K::kOffX + xs * kAtom;
                uint4 xv[8];
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) xv[c8] = *reinterpret_cast<const uint4*>(sx + swz(j, c8));
                // skip term into the Y'' accumulator (drained by the epilogue of item i - 3)
                tc_fence_after();
                {
                    const float2 d2 = make_float2(dq, dq);
#pragma unroll
                    for (int h4 = 0; h4 < 4; ++h4) {
                        uint32_t pre[16];
#pragma unroll
                        for (int cc = 0; cc < 2; ++cc) {
                            const uint32_t xw[4] = {xv[2 * h4 + cc].x, xv[2 * h4 + cc].y, xv[2 * h4 + cc].z,
                                                    xv[2 * h4 + cc].w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 v = mul2(d2, unpack_bf16(xw[e]));
                                pre[8 * cc + 2 * e] = __float_as_uint(v.x);
                                pre[8 * cc + 2 * e + 1] = __float_as_uint(v.y);
                            }
                        }
                        tmem_st16(tmem + lb + kColY + 64 * ys + 16 * h4, pre);
                    }
                    tmem_st_wait();
                }
                // w o x over the raw row (re-read: the unfactored path holds no copy)
                auto scale_in_place = [&]() {
                    const float2 w2 = make_float2(w, w);
#pragma unroll
                    for (int c8 = 0; c8 < 8; ++c8) {
                        const uint4 xr = *reinterpret_cast<const uint4*>(sx + swz(j, c8));
                        *reinterpret_cast<uint4*>(sx + swz(j, c8)) =
                            make_uint4(pack_bf16(mul2(w2, unpack_bf16(xr.x))), pack_bf16(mul2(w2, unpack_bf16(xr.y))),
                                       pack_bf16(mul2(w2, unpack_bf16(xr.z))), pack_bf16(mul2(w2, unpack_bf16(xr.w))));
                    }
                    fence_proxy_async_smem();
                };
                if (shared) {
                    scale_in_place();
                    if (j == 0) bs->xmode[xs] = 1;
                    tc_fence_before();
                    mbar_arrive(&bs->wx_full[xs]);
                } else {
                    // this head's P = G o exp(cs_j - cs_i) dt_i (exact exponent per element)
                    if (!wait_bar_all(&bs->p_empty, (pph & 1) ^ 1, bs, err)) goto done;
                    tc_fence_after();
                    __syncwarp();
                    const float* dts = cs + kTile;
#pragma unroll 1
                    for (int blk = 0; blk < 4; ++blk) {
                        uint32_t pk[16];
                        if (blk > wq) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) pk[e] = 0u;
                        } else {
                            float gv[32];
                            tmem_ld32(tmem + lb + kColG + 32 * blk, gv);
                            tmem_ld_wait_regs(gv);
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const int i0 = 32 * blk + 2 * e;
                                const float p0 = i0 <= j ? gv[2 * e] * ex2(csj - cs[i0]) * dts[i0] : 0.f;
                                const float p1 =
                                    i0 + 1 <= j ? gv[2 * e + 1] * ex2(csj - cs[i0 + 1]) * dts[i0 + 1] : 0.f;
                                pk[e] = pack_bf16(p0, p1);
                            }
                        }
                        tmem_st16(tmem + lb + kColP + 16 * blk, pk);
                    }
                    tmem_st_wait();
                    ++pph;
                    if (j == 0) bs->xmode[xs] = 0;
                    tc_fence_before();
                    mbar_arrive(&bs->wx_full[xs]);
                    if (k == kh - 1) mbar_arrive(&bs->g_empty);
                    // the product with the raw x tile has read it: now scale it in place
                    if (!wait_bar_all(&bs->xr_done, nsh & 1, bs, err)) goto done;
                    ++nsh;
                    scale_in_place();
                    mbar_arrive(&bs->wx2_full);
                }
                mbar_arrive(&bs->cs_empty[c]);
            }
        }
    } else if (warp >= 8 && warp < 16) {
        // ------------------------------------------------------------ chain group
        // Thread (q, lane) of warp 8 + 4 ph + q owns TMEM lane r = 32q + lane, i.e. state
        // row r (and r + 128), head-dim columns 32ph..32ph+31. Per item: the leaving
        // state 2^L h + S onto the chain, and the operand of C h^T (bf16 2^L h, or h)
        // into the item's operand buffer. The next item's entering state is loaded
        // while this one is finished.
        const int q = warp & 3;
        const int ph = (warp - 8) >> 2;
        const int r = q * 32 + lane;
        const uint32_t lb = (uint32_t)(q * 32) << 16;
        const int N = prm.N;
        constexpr bool kPrefetch = K::kMHalves == 1;
        float hv[32];
        bool have_h = false;          // hv holds the next item's entering state (row r)
        auto load_rows = [&](const float* src, int n, float (&v)[32]) {
            if (src && n < N) {
                const float* s0 = src + (int64_t)(32 * ph) * N + n;
#pragma unroll
                for (int p = 0; p < 32; ++p) v[p] = __ldcg(s0 + (int64_t)p * N);
            } else {
#pragma unroll
                for (int p = 0; p < 32; ++p) v[p] = 0.f;
            }
        };
        int np = 0;
        int m = 0, i = 0;
        for (;; ++m) {
            const int ur = m % kURing;
            if (!wait_bar_all(&bs->u_full[ur], (m / kURing) & 1, bs, err)) goto done;
            const int u = bs->uid[ur];
            mbar_arrive(&bs->u_empty[ur]);
            if (u < 0) break;
            const Unit U = decode(prm, u);
            for (int k = 0; k < kh; ++k, ++i) {
                const int ys = i % kYSlots, ss = i % K::kSSlots, hs = i % K::kHYSlots;
                const int h = U.hb * kh + k;
                if (!wait_bar_all(&bs->yi_full[ys], (i / kYSlots) & 1, bs, err)) goto done;
                const float* yi = reinterpret_cast<const float*>(smem + K::kOffYInfo + ys * kYInfoBytes);
                const float eL = yi[kTile];
                const bool shared = yi[kTile + 1] != 0.f;
                const float sc = shared ? eL : 1.f;   // the operand: 2^L h, or h
                const float* src = entry_src(prm, U, h);
                float* dst = chain_buf(prm, U, h);
                if (kPrefetch && !have_h) load_rows(src, r, hv);
                have_h = false;
                if (!wait_bar_all(&bs->hy_free[hs], ((i / K::kHYSlots) & 1) ^ 1, bs, err)) goto done;
                if (!wait_bar_all(&bs->s_full[ss], (i / K::kSSlots) & 1, bs, err)) goto done;
                if (!wait_bar_all(&bs->pub_empty[np % kPubStages], ((np / kPubStages) & 1) ^ 1, bs, err))
                    goto done;
                tc_fence_after();
                uint8_t* hy = smem + K::kOffHY + hs * K::kHYBytes;
#pragma unroll 1
                for (int mh = 0; mh < K::kMHalves; ++mh) {
                    const int n = r + 128 * mh;
                    if (!kPrefetch) load_rows(src, n, hv);
#pragma unroll
                    for (int pc = 0; pc < 2; ++pc) {   // 16 head-dim columns at a time
                        float sv[16];
                        tmem_ld16(tmem + lb + kColS + 64 * ss + 64 * mh + 32 * ph + 16 * pc, sv);
                        tmem_ld_wait_regs(sv);
                        if (n < N) {
                            float* d = dst + (int64_t)(32 * ph + 16 * pc) * N + n;
#pragma unroll
                            for (int e = 0; e < 16; ++e) __stcg(d + (int64_t)e * N, fmaf(eL, hv[16 * pc + e], sv[e]));
                        }
                        uint32_t op[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            op[e] = pack_bf16(sc * hv[16 * pc + 2 * e], sc * hv[16 * pc + 2 * e + 1]);
                        *reinterpret_cast<uint4*>(hy + swz(n, 4 * ph + 2 * pc)) = make_uint4(op[0], op[1], op[2], op[3]);
                        *reinterpret_cast<uint4*>(hy + swz(n, 4 * ph + 2 * pc + 1)) =
                            make_uint4(op[4], op[5], op[6], op[7]);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bs->h_full[hs]);
                if (shared) mbar_arrive(&bs->s_empty[ss]);
                mbar_arrive(&bs->pub_full[np % kPubStages]);
                ++np;
                // the next item of this unit: its entering state (its chain flag was
                // acquired before its Y'' info was published)
                if (kPrefetch && k + 1 < kh) {
                    const int yn = (i + 1) % kYSlots;
                    if (!wait_bar_all(&bs->yi_full[yn], ((i + 1) / kYSlots) & 1, bs, err)) goto done;
                    load_rows(entry_src(prm, U, h + 1), r, hv);
                    have_h = true;
                }
            }
        }
    } else if (warp >= 16) {
        // ------------------------------------------------------------ epilogue group
        // Thread (q, lane) of warp 16 + q owns token row r = 32q + lane (TMEM lane) and
        // all 64 head-dim columns: y = q_r Y'' (or Y'' + 2^cs_r R) staged in the warp's
        // own 4 KB (or, for the 256-wide state, over the item's operand buffer once the
        // state product has read it), then one TMA store of the warp's 32 rows.
        const int q = warp - 16;
        const int r = q * 32 + lane;
        const uint32_t lb = (uint32_t)(q * 32) << 16;
        int m = 0, i = 0;
        for (;; ++m) {
            const int ur = m % kURing;
            if (!wait_bar_all(&bs->u_full[ur], (m / kURing) & 1, bs, err)) goto done;
            const int u = bs->uid[ur];
            mbar_arrive(&bs->u_empty[ur]);
            if (u < 0) break;
            const Unit U = decode(prm, u);
            for (int k = 0; k < kh; ++k, ++i) {
                const int ys = i % kYSlots, ss = i % K::kSSlots, hs = i % K::kHYSlots;
                if (!wait_bar_all(&bs->y_full[ys], (i / kYSlots) & 1, bs, err)) goto done;
                tc_fence_after();
                const float* yi = reinterpret_cast<const float*>(smem + K::kOffYInfo + ys * kYInfoBytes);
                const float f = yi[r];
                const bool shared = yi[kTile + 1] != 0.f;
                const float2 f2 = make_float2(f, f);
                uint8_t* hy = K::kOwnStaging ? smem + K::kOffStage : smem + K::kOffHY + hs * K::kHYBytes;
                if (K::kOwnStaging) {
                    // the warp's previous store has read its staging rows
                    if (lane == 0) bulk_wait_group_read0();
                    __syncwarp();
                }
#pragma unroll 1
                for (int pc = 0; pc < 4; ++pc) {
                    float yv[16], rv[16];
                    tmem_ld16(tmem + lb + kColY + 64 * ys + 16 * pc, yv);
                    if (shared) {
                        tmem_ld_wait_regs(yv);
                    } else {
                        tmem_ld16(tmem + lb + kColS + 64 * ss + 16 * pc, rv);
                        tmem_ld_wait_regs(yv, rv);
                    }
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        uint32_t o[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {
                            const int x0 = 8 * cc + 2 * e2;
                            const float2 yy = make_float2(yv[x0], yv[x0 + 1]);
                            o[e2] = pack_bf16(shared ? mul2(f2, yy) : fma2(f2, make_float2(rv[x0], rv[x0 + 1]), yy));
                        }
                        *reinterpret_cast<uint4*>(hy + swz(r, 2 * pc + cc)) = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
                tc_fence_before();
                mbar_arrive(&bs->y_empty[ys]);
                if (!shared) mbar_arrive_cnt(&bs->s_empty[ss], 2);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    if (U.t0 + 32 * q < T) {   // rows past T are clipped by the store
                        tma_store_4d(&tm_y, hy + q * (kAtom / 4), 0, U.hb * kh + k, (int)(U.t0 + 32 * q), U.b);
                        bulk_commit_group();
                        if (!K::kOwnStaging) bulk_wait_group_read0();
                    }
                    if (!K::kOwnStaging) mbar_arrive(&bs->hy_free[hs]);
                }
                __syncwarp();
            }
        }
    }
done:
    // y stores finish before the CTA exits
    if (warp >= 16 && lane == 0) bulk_wait_group0();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

int num_sms() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

template <int NS>
cudaError_t launch_ns(const FusedLaunch& a, const Params& prm, cudaStream_t st) {
    using K = Cfg<NS>;
    cudaError_t e = cudaFuncSetAttribute(ssd_fused_kernel<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)K::kSmem);
    if (e != cudaSuccess) return e;
    const int sms = num_sms();
    const int grid = prm.nunits < sms ? prm.nunits : sms;
    ssd_fused_kernel<NS><<<grid, kThreads, K::kSmem, st>>>(a.maps[0], a.maps[1], a.maps[2], a.maps[3], prm);
    return cudaGetLastError();
}

}  // namespace

int fused_state_capacity(int64_t N) {
    if (N < 16 || N % 16 != 0) return 0;
    if (N <= 128) return 128;
    if (N <= 256) return 256;
    return 0;
}

int fused_kheads(int64_t H, int64_t G, int ns) {
    const int64_t hpg = H / G;
    const int want = ns == 256 ? 8 : 4;
    for (int k = want; k > 1; --k)
        if (hpg % k == 0) return k;
    return 1;
}

size_t fused_sync_ints(const Dims& d, int nseg) { return 2 + (size_t)(d.b * nseg * d.H); }

cudaError_t launch_fused(const FusedLaunch& a, cudaStream_t st) {
    const Dims& d = a.d;
    cudaError_t e = cudaMemsetAsync(a.sync_ints, 0, sizeof(int) * fused_sync_ints(d, a.nseg), st);
    if (e != cudaSuccess) return e;
    const int ns = fused_state_capacity(d.N);
    if (ns == 0 || a.nseg < 1 || a.seg_tiles < 1) return cudaErrorInvalidValue;
    Params prm = {};
    prm.dt = a.dt;
    prm.A = a.A;
    prm.D = a.D;
    prm.init = a.init;
    prm.finalbuf = a.finalbuf;
    prm.segbuf = a.segbuf;
    prm.ticket = a.sync_ints;
    prm.error = a.sync_ints + 1;
    prm.flags = a.sync_ints + 2;
    prm.T = d.T;
    prm.H = (int)d.H;
    prm.G = (int)d.G;
    prm.N = (int)d.N;
    prm.kheads = a.kheads;
    prm.batch = (int)d.b;
    const int64_t ntiles = (d.T + kTile - 1) / kTile;
    const int64_t nunits = (int64_t)a.seg_tiles * a.nseg * d.b * (d.H / a.kheads);
    if (nunits > INT32_MAX / 2 || d.T > INT32_MAX || (int64_t)a.seg_tiles * a.nseg < ntiles)
        return cudaErrorInvalidValue;
    prm.nunits = (int)nunits;
    prm.ntiles = (int)ntiles;
    prm.seg_tiles = a.seg_tiles;
    prm.nseg = a.nseg;
    prm.stall = a.stall;
    return ns == 128 ? launch_ns<128>(a, prm, st) : launch_ns<256>(a, prm, st);
}

}  // namespace ssd
