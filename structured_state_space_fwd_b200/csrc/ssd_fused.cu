// Warp-specialized, persistent single-pass SSD forward for sm_100a.
//
// "Transformers are SSMs" (Knowl 1, 2, 3, 7) in 128-token tiles: per tile the
// diagonal block in the quadratic masked form, everything before the tile
// through the state entering it. With cs the inclusive cumulative sum of dt*A
// inside the tile (log2 units), L = cs of the tile's last token,
// w_i = 2^(L - cs_i) dt_i and q_j = 2^(cs_j - L), a tile's outputs and the
// state leaving it are
//
//   y_j  = q_j [ (tril(C B^T) (w o x))_j + C_j . (2^L h) + D x_j / q_j ]
//   h'   = 2^L h + B^T (w o x)
//
// (the 1-semiseparable mask of Knowl 3 factored through the tile's last token).
// The three terms in brackets accumulate in ONE tensor-memory accumulator Y'':
// the skip term is stored into it first, then the masked product and the state
// term are added by the tensor cores, so the epilogue is one scaling. A tile
// whose heads decay by more than 2^96 over it takes the unfactored form:
// per head P = (C B^T) o exp(segsum) o dt (exponent per element), Y = P x + D x,
// R = C h^T in a separate accumulator, y = Y + 2^cs R.
//
// Work unit: a SEGMENT of up to `seg_tiles` consecutive tiles of one batch row
// and one pair of heads of a group (Knowl 7: the pair shares B and C). The CTA
// that takes a unit walks its tiles in order and carries the pair's state in
// registers from tile to tile (Knowl 2's state passing, inside the unit); only
// the state entering the unit and the state leaving it touch global memory.
// Every product of a tile is one MMA group of N = 128 (the two heads' 64
// columns side by side). The state entering segment s > 0 is written by the
// unit of segment s - 1 (units are handed out by an atomic ticket in
// segment-major order, so that unit was taken earlier by a running CTA, and a
// flag says when its state is out), or, for sequences with few (batch row,
// pair) chains, computed beforehand by the segment-state pass and the scan over
// segments (ssd_segment.cu), so that all segments run at once.
//
// Roles (20 warps):
//   warp 0      TMA producer; takes units from the ticket and hands their ids to
//               every role through a small ring
//   warp 1      TMEM owner and MMA issuer (one thread)
//   warp 2      per tile and head: dt loads, cumulative sum
//   warp 3      per unit: makes the leaving state visible and releases its flag
//   warps 4-7   mask group (thread = token row): per tile tril(C B^T) into TMEM,
//               the skip-term preload and w o x in place of the x tiles
//   warps 8-15  chain group (thread = state row, half of the head dim): per unit
//               the flag of the state entering it (acquire) and that state; carries
//               the state, per tile the bf16 operand of C (2^L h)^T
//   warps 16-19 epilogue group (thread = token row): per tile and head
//               y = q Y'', staged in shared memory (optionally gated by SiLU(z)
//               and RMS-normalised over groups within the head), one TMA store
//               per warp
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
constexpr int kCsSlots = 4;       // per tile and head
constexpr int kYSlots = 2;        // Y'' accumulators, one tile of the pair each
constexpr int kURing = 4;

constexpr uint32_t kAtom = kTile * 128;    // 16 KB: 128 rows of 128 bytes (64 bf16)
// per tile and head: cs[128], dt[128], then L (cs of the last token), D_h, tile mode
constexpr uint32_t kCsSlotBytes = 2 * kTile * 4 + 64;
constexpr int kCsL = 2 * kTile, kCsD = 2 * kTile + 1, kCsMode = 2 * kTile + 2;
// per Y'' accumulator: each head's row factor (q_j, or 2^cs_j), per head 2^L, the mode
constexpr uint32_t kYInfoBytes = 2 * kTile * 4 + 16;
constexpr int kYiEL = 2 * kTile, kYiMode = 2 * kTile + 2;

// TMEM columns: G = C B^T (fp32), overwritten in place by P' = tril(G) (bf16
// pairs, columns 0..63) for factored tiles; the S slot (the pair's two 64-column
// states, or one 256-row state as two halves; for an unfactored tile first its
// per-head P, later its C h^T); two Y'' accumulators of a pair each.
constexpr uint32_t kColG = 0;
constexpr uint32_t kColP = 0;
constexpr uint32_t kColS = 128;
constexpr uint32_t kColY = 256;

constexpr float kLog2e = 1.4426950408889634f;
// Widest decay over one tile (log2 units) for which a tile takes the factored
// form: 2^(L - cs) dt (bf16 operand) and 2^(L - cs) (skip-term divisor) then stay
// inside the normal fp32 / bf16 exponent range with a wide margin.
constexpr float kSharedMaskRangeLog2 = 96.f;

// Shared-memory layout for state capacity NS (128 or 256 state elements). B and C
// tiles live in a ring of tile buffers taken in the order B_0, C_0, B_1, C_1, ...:
// a tile's B is released once its S product is done, its C once its state
// product is.
template <int NS>
struct Cfg {
    static constexpr int kAtoms = NS / 64;                  // 64-wide column atoms of B or C
    static constexpr uint32_t kBCTile = kAtoms * kAtom;     // B (or C) tile
    static constexpr int kBufs = NS == 128 ? 3 : 2;         // tile buffers
    static constexpr int kMH = NS / 128;                    // 128-row halves of the state
    static constexpr int kNP = NS == 128 ? 2 : 1;           // heads per unit at most
    static constexpr int kXSlots = 2;                       // x slots, one tile of the pair each
    static constexpr uint32_t kXBytes = kNP * kAtom;
    static constexpr uint32_t kHBytes = 2 * kAtom;          // state operand: 2 atoms
    static constexpr uint32_t kOffBC = 0;
    static constexpr uint32_t kOffX = kOffBC + kBufs * kBCTile;
    static constexpr uint32_t kOffH = kOffX + kXSlots * kXBytes;
    static constexpr uint32_t kOffStage = kOffH + kHBytes;  // 4 KB per epilogue warp
    static constexpr uint32_t kOffCs = kOffStage + kAtom;
    static constexpr uint32_t kOffYInfo = kOffCs + kCsSlots * kCsSlotBytes;
    static constexpr uint32_t kOffBar = kOffYInfo + kYSlots * kYInfoBytes;
    static constexpr uint32_t kSmem = kOffBar + 1024;
    static_assert(kSmem <= 232448, "shared memory budget");
};

struct Params {
    const float* dt;
    const float* A;
    const float* D;
    const float* init;    // [b,H,P,N] or null (zeros)
    float* finalbuf;      // [b,H,P,N] final states, or null (not written)
    float* segbuf;        // [b,nseg,H,P,N]: slot s >= 1 holds the state entering segment s
    int* ticket;
    int* error;
    int* flags;           // [b*nseg*nhb] state entering the segment written (chained)
    void* y;              // [b,T,H,P] bf16 (the gated output when z is set), for rows a
                          // tile store must not cover
    const __nv_bfloat16* z;   // gate branch [b,T,H,P] bf16, or null: y is stored as is
    const float* nw;      // norm weight [H*P] fp32 (with z)
    int gs;               // norm group size, dividing 64 and a multiple of 8 (with z)
    float eps;            // norm epsilon (with z)
    const int* cu;        // packed documents: token offsets [ndoc+1] in batch row 0, or null
    const int* order;     // packed documents: unit order (documents, longest first)
    int64_t T;
    int H, G, N, kheads, batch, nunits, ntiles, seg_tiles, nseg;
    int seg_first;        // tiles of segment 0 (the others: seg_tiles)
    int nslot;            // segbuf slots per batch row (nseg, or more)
    int chained;          // entering states come from the previous segment's unit
    int stall;            // test builds only: chain flags awaited at a value never reached
};

struct Bars {
    uint64_t u_full[kURing], u_empty[kURing];
    uint64_t tb_full[3], tb_empty[3];
    uint64_t x_full[2], x_empty[2];
    uint64_t wx_full[2];          // tile's operands ready (w o x, or per-head P and raw x); mode in xmode
    uint64_t wx2_full;            // unfactored tile: x scaled in place after Y = P x
    uint64_t xr_done;             // unfactored tile: Y = P x has read the raw tiles
    uint64_t g_full, g_empty_mma, g_empty_mask, p_full;
    uint64_t cs_full[kCsSlots], cs_empty[kCsSlots];
    uint64_t s_full, s_empty;
    uint64_t s_read;              // unfactored tile: the chain group has read S (its slot takes C h^T next)
    uint64_t y_full[kYSlots], y_empty[kYSlots], yi_full[kYSlots];
    uint64_t h_full, h_free;
    uint64_t pub_full[2], pub_empty[2];   // per unit: leaving state stored / flag released
    uint64_t fin;
    int uid[kURing];
    int xmode[2];
    uint32_t tmem;
    int abort;
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

// arrivals on u_empty: x loader, MMA thread, cumsum warp, publisher, mask, chain and
// epilogue groups
constexpr uint32_t kUnitReaders = 1 + 1 + 32 + 1 + 128 + 256 + 128;

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Orders every memory access this thread has made or observed (the chain group's
// state stores, seen through an mbarrier) before its later accesses, GPU-wide.
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
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
    int s, b, hb;          // segment, batch row, head block (pair)
    int t_begin, t_end;    // its tiles
    int doc;               // sequence index of the initial / final states (batch row, or document)
    int tok0, len;         // the sequence's first token in its row, its length in tokens
};
__device__ __forceinline__ Unit decode(const Params& p, int u) {
    const int nhb = p.H / p.kheads;
    Unit r;
    r.hb = u % nhb;
    int q = u / nhb;
    if (p.cu) {
        // packed documents: one unit per (document, head block), the whole document;
        // offsets are clamped to the row, so a malformed list reads and writes only
        // inside it (the ordering kernel reports it)
        r.doc = __ldg(p.order + q);
        const int a = min(max(__ldg(p.cu + r.doc), 0), (int)p.T);
        const int e = min(max(__ldg(p.cu + r.doc + 1), a), (int)p.T);
        r.b = 0;
        r.s = 0;
        r.tok0 = a;
        r.len = e - a;
        r.t_begin = 0;
        r.t_end = (r.len + kTile - 1) / kTile;
        return r;
    }
    r.b = q % p.batch;
    r.s = q / p.batch;
    r.doc = r.b;
    r.tok0 = 0;
    r.len = (int)p.T;
    r.t_begin = r.s == 0 ? 0 : p.seg_first + (r.s - 1) * p.seg_tiles;
    r.t_end = min(p.ntiles, r.s == 0 ? p.seg_first : r.t_begin + p.seg_tiles);
    return r;
}
__device__ __forceinline__ int64_t flag_index(const Params& p, int b, int s, int hb) {
    return ((int64_t)b * p.nseg + s) * (p.H / p.kheads) + hb;
}
// Waits (bounded) for the flag of the state entering a chained unit and acquires
// it; false (error word and abort set) when the wait runs out.
__device__ __forceinline__ bool acquire_entry_flag(const Params& p, const Unit& U, Bars* bs, int* err) {
    const int* f = p.flags + flag_index(p, U.b, U.s, U.hb);
    const int want = 1 + (p.stall ? (1 << 30) : 0);
    const uint64_t t0 = global_ns();
    for (uint32_t it = 0;; ++it) {
        if (ld_acquire(f) >= want) return true;
        if (it >= 2) __nanosleep(128);
        if ((it & 15) == 15 && (*(volatile int*)&bs->abort || global_ns() - t0 > kWaitLimitNs)) break;
    }
    *(volatile int*)&bs->abort = 1;
    atomicExch(err, 1);
    return false;
}
// state entering the unit for head h (null: zeros)
__device__ __forceinline__ const float* entry_src(const Params& p, const Unit& U, int h) {
    const int64_t PN = (int64_t)kP * p.N;
    if (U.s == 0) return p.init ? p.init + ((int64_t)U.doc * p.H + h) * PN : nullptr;
    return p.segbuf + (((int64_t)U.b * p.nslot + U.s) * p.H + h) * PN;
}
// where the state leaving the unit goes for head h (null: nowhere)
__device__ __forceinline__ float* exit_dst(const Params& p, const Unit& U, int h) {
    const int64_t PN = (int64_t)kP * p.N;
    if (U.s == p.nseg - 1) return p.finalbuf ? p.finalbuf + ((int64_t)U.doc * p.H + h) * PN : nullptr;
    if (!p.chained) return nullptr;
    return p.segbuf + (((int64_t)U.b * p.nslot + U.s + 1) * p.H + h) * PN;
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
// ks: 1, 2, 4 or 8 with a state capacity of 128; always 16 with 256 (a state above 128)
template <bool kBRows, int NS>
__device__ __forceinline__ void mma_state_dim_n(int ks, uint32_t d, uint64_t dA, uint64_t dB, uint32_t idesc,
                                                uint32_t acc0) {
    if constexpr (NS == 256) {
        mma_state_dim<16, kBRows>(d, dA, dB, idesc, acc0);
    } else {
        switch (ks) {
            case 1: mma_state_dim<1, kBRows>(d, dA, dB, idesc, acc0); break;
            case 2: mma_state_dim<2, kBRows>(d, dA, dB, idesc, acc0); break;
            case 4: mma_state_dim<4, kBRows>(d, dA, dB, idesc, acc0); break;
            case 8: mma_state_dim<8, kBRows>(d, dA, dB, idesc, acc0); break;
            default: mma_state_dim<16, kBRows>(d, dA, dB, idesc, acc0); break;
        }
    }
}
// 8 steps of K = 16 over the tile's tokens: A from shared memory (B^T, N-contiguous)
// or from tensor memory (P), B the x tiles of the pair (N-contiguous).
__device__ __forceinline__ void mma_tokens_smem(uint32_t d, uint64_t dA, uint64_t dB, uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < kTile / 16; ++kk)
        mma_bf16(d, dA + (uint64_t)(kk * 128), dB + (uint64_t)(kk * 128), idesc, kk > 0 ? 1u : 0u);
}
__device__ __forceinline__ void mma_tokens_tmem(uint32_t d, uint32_t a, uint64_t dB, uint32_t idesc) {
#pragma unroll
    for (int kk = 0; kk < kTile / 16; ++kk)
        mma_bf16_tmem_a(d, a + 8 * kk, dB + (uint64_t)(kk * 128), idesc, 1u);
}

// The skip term D x_j / q_j (or D x_j) of one head into its 64 columns of the
// tile's Y'' (taddr: this warp's lanes, the head's first column), from the thread's
// bf16 row of x.
__device__ __forceinline__ void preload_skip(uint32_t taddr, const uint4 (&xv)[8], float dq) {
    const float2 d2 = make_float2(dq, dq);
#pragma unroll
    for (int h4 = 0; h4 < 4; ++h4) {
        uint32_t pre[16];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const uint32_t xw[4] = {xv[2 * h4 + cc].x, xv[2 * h4 + cc].y, xv[2 * h4 + cc].z, xv[2 * h4 + cc].w};
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
                const float2 v = mul2(d2, unpack_bf16(xw[e2]));
                pre[8 * cc + 2 * e2] = __float_as_uint(v.x);
                pre[8 * cc + 2 * e2 + 1] = __float_as_uint(v.y);
            }
        }
        tmem_st16(taddr + 16 * h4, pre);
    }
}

// The mask group's work on a tile in the unfactored form (a head decays by more than
// 2^96 over it), for thread j (token row j, TMEM lanes at tl = tmem base + lane
// quarter): per head the skip term, the row's factor 2^cs_j, and its
// P = G o exp(cs_j - cs_i) dt_i (exponent per element) in the S slot; then, after the
// products with the raw x tiles, w o x in place. Kept out of line: it is rare, and
// its registers would otherwise weigh on the common path. False if a wait gave up.
__device__ __noinline__ bool mask_unfactored_tile(Bars* bs, int* err, const float* cs_base, float* yi,
                                                  uint8_t* sxp, uint32_t tl, int ys, int xs, int hi, int np,
                                                  int i, int nsh, int j, int wq) {
    // the per-head masks need G and go into the S slot (free once the previous tile's
    // S, or C h^T, has been read)
    if (!wait_bar_all(&bs->g_full, i & 1, bs, err)) return false;
    if (!wait_bar_all(&bs->s_empty, (i & 1) ^ 1, bs, err)) return false;
    tc_fence_after();
    __syncwarp();
    float wv[2];
    for (int e = 0; e < np; ++e) {
        const int c = (hi + e) % kCsSlots;
        if (!wait_bar_all(&bs->cs_full[c], ((hi + e) / kCsSlots) & 1, bs, err)) return false;
        const float* cs = cs_base + c * (kCsSlotBytes / 4);
        const float L = cs[kCsL], csj = cs[j];
        wv[e] = ex2(L - csj) * cs[kTile + j];
        yi[e * kTile + j] = ex2(csj);
        if (j == 0) yi[kYiEL + e] = ex2(L);
        uint8_t* sx = sxp + e * kAtom;
        uint4 xv[8];
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) xv[c8] = *reinterpret_cast<const uint4*>(sx + swz(j, c8));
        preload_skip(tl + kColY + 128 * ys + 64 * e, xv, cs[kCsD]);
        const float* dts = cs + kTile;
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
            uint32_t pk[16];
            if (blk > wq) {
#pragma unroll
                for (int q2 = 0; q2 < 16; ++q2) pk[q2] = 0u;
            } else {
                float gv[32];
                tmem_ld32(tl + kColG + 32 * blk, gv);
                tmem_ld_wait_regs(gv);
#pragma unroll
                for (int q2 = 0; q2 < 16; ++q2) {
                    const int i0 = 32 * blk + 2 * q2;
                    const float p0 = i0 <= j ? gv[2 * q2] * ex2(csj - cs[i0]) * dts[i0] : 0.f;
                    const float p1 = i0 + 1 <= j ? gv[2 * q2 + 1] * ex2(csj - cs[i0 + 1]) * dts[i0 + 1] : 0.f;
                    pk[q2] = pack_bf16(p0, p1);
                }
            }
            tmem_st16(tl + kColS + 64 * e + 16 * blk, pk);
        }
    }
    if (j == 0) yi[kYiMode] = 0.f;
    tmem_st_wait();
    mbar_arrive(&bs->yi_full[ys]);
    if (j == 0) bs->xmode[xs] = 0;
    tc_fence_before();
    mbar_arrive(&bs->wx_full[xs]);
    mbar_arrive(&bs->g_empty_mask);     // G has served the masks
    // the products with the raw x tiles have read them: now scale in place
    if (!wait_bar_all(&bs->xr_done, nsh & 1, bs, err)) return false;
    for (int e = 0; e < np; ++e) {
        uint8_t* sx = sxp + e * kAtom;
        const float2 w2 = make_float2(wv[e], wv[e]);
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
            const uint4 xr = *reinterpret_cast<const uint4*>(sx + swz(j, c8));
            *reinterpret_cast<uint4*>(sx + swz(j, c8)) =
                make_uint4(pack_bf16(mul2(w2, unpack_bf16(xr.x))), pack_bf16(mul2(w2, unpack_bf16(xr.y))),
                           pack_bf16(mul2(w2, unpack_bf16(xr.z))), pack_bf16(mul2(w2, unpack_bf16(xr.w))));
        }
    }
    fence_proxy_async_smem();
    mbar_arrive(&bs->wx2_full);
    return true;
}

// The MMA issuer's work on a tile in the unfactored form, after G: per head Y = P x
// with the raw x tile (P in the S slot), S once the tile is scaled in place, and C h^T
// into the S slot once the chain group has read S. Out of line for the same reason
// as the mask group's. False if a wait gave up.
template <int NS>
__device__ __noinline__ bool mma_unfactored_tile(Bars* bs, int* err, uint32_t tmem, int ys, int xs, int tbB,
                                                 int tbC, int item, int nsh, int nrd, int np, int kmh, int ksN,
                                                 uint64_t dX, uint64_t dSA, uint64_t dC, uint64_t dH, uint32_t idS,
                                                 uint32_t idY) {
    constexpr uint32_t idY1 = idesc_bf16(128, 64, 0, 1);   // one head
    tc_fence_after();
    for (int e = 0; e < np; ++e)
        mma_tokens_tmem(tmem + kColY + 128 * ys + 64 * e, tmem + kColS + 64 * e, dX + (uint64_t)((e * kAtom) >> 4),
                        idY1);
    mma_commit(&bs->xr_done);
    if (!wait_bar(&bs->wx2_full, nsh & 1, bs, err)) return false;
    tc_fence_after();
    for (int mh = 0; mh < kmh; ++mh)
        mma_tokens_smem(tmem + kColS + 64 * mh, dSA + (uint64_t)((2 * mh * kAtom) >> 4), dX, idS);
    mma_commit(&bs->s_full);
    mma_commit(&bs->x_empty[xs]);
    mma_commit(&bs->tb_empty[tbB]);    // this tile's B has served G and S
    if (!wait_bar(&bs->s_read, nrd & 1, bs, err)) return false;
    if (!wait_bar(&bs->h_full, item & 1, bs, err)) return false;
    tc_fence_after();
    mma_state_dim_n<true, NS>(ksN, tmem + kColS, dC, dH, idY, 0u);
    mma_commit(&bs->h_free);
    mma_commit(&bs->tb_empty[tbC]);
    mma_commit(&bs->y_full[ys]);
    return true;
}

// The epilogue's row of an unfactored tile for head e: y = Y'' + f R (f = 2^cs_r, R
// in the S slot), bf16 into the staging row r. Out of line, as the rest of that form.
__device__ __noinline__ void stage_unfactored_row(uint32_t tl, int ys, int e, float f, uint8_t* stg, int r) {
    const float2 f2 = make_float2(f, f);
#pragma unroll 1
    for (int pc = 0; pc < 4; ++pc) {
        float yv[16], rv[16];
        tmem_ld16(tl + kColY + 128 * ys + 64 * e + 16 * pc, yv);
        tmem_ld16(tl + kColS + 64 * e + 16 * pc, rv);
        tmem_ld_wait_regs(yv, rv);
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            uint32_t o[4];
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
                const int x0 = 8 * cc + 2 * e2;
                o[e2] = pack_bf16(fma2(f2, make_float2(rv[x0], rv[x0 + 1]), make_float2(yv[x0], yv[x0 + 1])));
            }
            *reinterpret_cast<uint4*>(stg + swz(r, 2 * pc + cc)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// SiLU(z) = z sigmoid(z) = z (1 + tanh(z / 2)) / 2: one special-function
// instruction (tanh.approx, a relative error near 2^-11, under the bf16 output's
// rounding).
__device__ __forceinline__ float silu_fast(float z) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
    return 0.5f * z * (1.f + t);
}

// One group size's pass of gate_row below: v is held in registers between the sum
// of squares and the scaling for groups of up to 32 channels, recomputed for 64.
template <int GC>   // 16-byte chunks (8 channels) per group
__device__ __forceinline__ void gate_row_g(const uint4 (&zv)[8], const float* w, float eps, uint8_t* stg, int r) {
    constexpr float kInvGs = 1.f / (8 * GC);
    auto gated = [&](int c, float (&v)[8]) {
        const uint4 yv = *reinterpret_cast<const uint4*>(stg + swz(r, c));
        const uint32_t ys4[4] = {yv.x, yv.y, yv.z, yv.w};
        const uint32_t zs4[4] = {zv[c].x, zv[c].y, zv[c].z, zv[c].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 y2 = unpack_bf16(ys4[k]), z2 = unpack_bf16(zs4[k]);
            v[2 * k] = y2.x * silu_fast(z2.x);
            v[2 * k + 1] = y2.y * silu_fast(z2.y);
        }
    };
#pragma unroll
    for (int c0 = 0; c0 < 8; c0 += GC) {
        constexpr int kHold = GC <= 4 ? GC : 1;   // chunks whose v stays in registers
        float vh[kHold][8];
        float ss = 0.f;
#pragma unroll
        for (int c = c0; c < c0 + GC; ++c) {
            float v[8];
            gated(c, v);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                ss = fmaf(v[k], v[k], ss);
                if (GC <= 4) vh[(c - c0) % kHold][k] = v[k];
            }
        }
        const float inv = rsqrtf(ss * kInvGs + eps);
#pragma unroll
        for (int c = c0; c < c0 + GC; ++c) {
            float v[8];
            if (GC <= 4) {
#pragma unroll
                for (int k = 0; k < 8; ++k) v[k] = vh[(c - c0) % kHold][k];
            } else {
                gated(c, v);
            }
            const float4 w0 = __ldg(reinterpret_cast<const float4*>(w + 8 * c));
            const float4 w1 = __ldg(reinterpret_cast<const float4*>(w + 8 * c + 4));
            const float wk[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) o[k] = pack_bf16(v[2 * k] * inv * wk[2 * k], v[2 * k + 1] * inv * wk[2 * k + 1]);
            *reinterpret_cast<uint4*>(stg + swz(r, c)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}
// The gate and normalisation after the layer ("Transformers are SSMs", Knowl 6,
// step 4) on one staged row of 64 channels (head hh of one token, bf16 y in the
// 128-byte-swizzled staging row r), in place: v = y * SiLU(z), then each group
// of gs channels is divided by sqrt(mean(v^2) + eps) and scaled by the weight.
// y is the bf16 value a separate pass would read back. zrow indexes [b,T,H] of z.
__device__ __noinline__ void gate_row(const __nv_bfloat16* z, const float* nw, int gs, float eps, uint8_t* stg,
                                     int r, int64_t zrow, int hh) {
    const uint4* zp = reinterpret_cast<const uint4*>(z + zrow * kP);
    uint4 zv[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) zv[c] = __ldg(zp + c);    // each 32-byte sector over two loads: via L1
    const float* w = nw + (int64_t)hh * kP;
    switch (gs) {
        case 8: gate_row_g<1>(zv, w, eps, stg, r); break;
        case 16: gate_row_g<2>(zv, w, eps, stg, r); break;
        case 32: gate_row_g<4>(zv, w, eps, stg, r); break;
        default: gate_row_g<8>(zv, w, eps, stg, r); break;
    }
}

template <int NS, bool kGate>
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
            mbar_init(&bs->x_full[i], 1);
            mbar_init(&bs->x_empty[i], 1);
            mbar_init(&bs->wx_full[i], 128);
            mbar_init(&bs->pub_full[i], 256);
            mbar_init(&bs->pub_empty[i], 1);
        }
        mbar_init(&bs->wx2_full, 128);
        mbar_init(&bs->xr_done, 1);
        mbar_init(&bs->g_full, 1);
        mbar_init(&bs->g_empty_mma, 1);
        mbar_init(&bs->g_empty_mask, 128);
        mbar_init(&bs->p_full, 128);
        for (int i = 0; i < kCsSlots; ++i) {
            mbar_init(&bs->cs_full[i], 32);
            mbar_init(&bs->cs_empty[i], 128);
        }
        mbar_init(&bs->s_full, 1);
        mbar_init(&bs->s_empty, 256);
        mbar_init(&bs->s_read, 256);
        for (int i = 0; i < kYSlots; ++i) {
            mbar_init(&bs->y_full[i], 1);
            mbar_init(&bs->y_empty[i], 128);
            mbar_init(&bs->yi_full[i], 128);
        }
        mbar_init(&bs->h_full, 256);
        mbar_init(&bs->h_free, 1);
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
    const int np = prm.kheads;             // heads per unit (1 or 2)
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
        // Lane 0 takes units and loads B and C; lane 1 loads the x tiles, so that they
        // do not queue behind tile buffers still in use.
        if (lane == 1) {
            int n = 0;
            for (int m = 0;; ++m) {
                const int ur = m % kURing;
                if (!wait_bar_idle(&bs->u_full[ur], (m / kURing) & 1, bs, err)) goto xdrain;
                const int u = bs->uid[ur];
                mbar_arrive(&bs->u_empty[ur]);
                if (u < 0) break;
                const Unit U = decode(prm, u);
                for (int t = U.t_begin; t < U.t_end; ++t, ++n) {
                    const int xs = n % K::kXSlots;
                    if (!wait_bar_idle(&bs->x_empty[xs], ((n / K::kXSlots) & 1) ^ 1, bs, err)) goto xdrain;
                    mbar_arrive_expect_tx(&bs->x_full[xs], np * kAtom);
                    for (int e = 0; e < np; ++e)
                        tma_load_4d(smem + K::kOffX + xs * K::kXBytes + e * kAtom, &tm_x, &bs->x_full[xs], 0,
                                    U.hb * np + e, U.tok0 + t * kTile, U.b);
                }
            }
        xdrain:
            for (int i = 0; i < K::kXSlots && i < n; ++i)
                mbar_wait(&bs->x_full[(n - 1 - i) % K::kXSlots], ((n - 1 - i) / K::kXSlots) & 1, 1u << 22);
        } else if (lane == 0) {
            int mb = 0;    // tile buffers loaded
            auto take = [&]() -> int {
                int u;
                do {
                    u = atomicAdd(prm.ticket, 1);
                } while (u < prm.nunits && decode(prm, u).t_begin >= prm.ntiles);
                return u < prm.nunits ? u : -1;
            };
            auto publish = [&](int m, int u) -> bool {
                const int ur = m % kURing;
                if (!wait_bar_idle(&bs->u_empty[ur], ((m / kURing) & 1) ^ 1, bs, err)) return false;
                bs->uid[ur] = u;
                mbar_arrive(&bs->u_full[ur]);
                return true;
            };
            // Each unit's successor is taken and published before the unit's own tiles
            // are loaded, so the other roles (the x loader first) run into it without
            // waiting for this lane. Units are still taken in ticket order and worked in
            // that order, so a chained unit's predecessor always has a lower ticket that
            // some CTA is working on or has finished.
            int u = take();
            if (!publish(0, u)) goto pdrain;
            for (int m = 0; u >= 0; ++m) {
                const int un = take();
                if (!publish(m + 1, un)) goto pdrain;
                const Unit U = decode(prm, u);
                const int g = U.hb * np / (H / prm.G);
                for (int t = U.t_begin; t < U.t_end; ++t) {
                    for (int bc = 0; bc < 2; ++bc, ++mb) {    // B, then C
                        const int tb = mb % K::kBufs;
                        if (!wait_bar_idle(&bs->tb_empty[tb], ((mb / K::kBufs) & 1) ^ 1, bs, err)) goto pdrain;
                        mbar_arrive_expect_tx(&bs->tb_full[tb], natoms * kAtom);
                        for (int a = 0; a < natoms; ++a)
                            tma_load_4d(smem + K::kOffBC + tb * K::kBCTile + a * kAtom, bc ? &tm_C : &tm_B,
                                        &bs->tb_full[tb], a * 64, g, U.tok0 + t * kTile, U.b);
                    }
                }
                u = un;
            }
        pdrain:
            // No TMA load may still be writing shared memory when the CTA exits: wait for
            // the last load issued into each buffer (already complete unless a role aborted).
            for (int i = 0; i < K::kBufs && i < mb; ++i)
                mbar_wait(&bs->tb_full[(mb - 1 - i) % K::kBufs], ((mb - 1 - i) / K::kBufs) & 1, 1u << 22);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Per tile i (factored): G = C B^T, S_i, the state term C (2^L h)^T once the
        // chain group has written its operand from the state entering the tile (ready
        // a tile ahead: it needs S_{i-1}, not S_i), then the masked product. An
        // unfactored tile: per-head Y = P x, S_i, and C h^T into the S slot once the
        // chain group has read S_i.
        if (lane == 0) {
            constexpr uint32_t idG = idesc_bf16(128, 128, 0, 0);   // C (K-major) x B (K-major)
            const uint32_t idS = np == 2 ? idesc_bf16(128, 128, 1, 1) : idesc_bf16(128, 64, 1, 1);
            const uint32_t idY = np == 2 ? idesc_bf16(128, 128, 0, 1) : idesc_bf16(128, 64, 0, 1);
            const uint64_t dH = sw128_desc(smem_u32(smem + K::kOffH), kAtom, 1024);
            struct Pend {
                int item, ys, cb;   // cb: tile buffer of the tile's C
                bool shared;
            };
            int psh = 0, nsh = 0, nrd = 0, gm = 0, gk = 0;
            bool prev_shared = true;
            // C (2^L h)^T onto Y'' (factored) or C h^T into the S slot (unfactored)
            auto issue_r = [&](const Pend& q) -> bool {
                if (!wait_bar(&bs->h_full, q.item & 1, bs, err)) return false;
                tc_fence_after();
                const uint64_t dC = sw128_desc(smem_u32(smem + K::kOffBC + q.cb * K::kBCTile), 16, 1024);
                const uint32_t d = q.shared ? tmem + kColY + 128 * q.ys : tmem + kColS;
                mma_state_dim_n<true, NS>(ksN, d, dC, dH, idY, q.shared ? 1u : 0u);
                mma_commit(&bs->h_free);
                mma_commit(&bs->tb_empty[q.cb]);
                return true;
            };
            int m = 0, i = 0;
            for (;; ++m) {
                const int ur = m % kURing;
                if (!wait_bar(&bs->u_full[ur], (m / kURing) & 1, bs, err)) goto drain;
                const int u = bs->uid[ur];
                mbar_arrive(&bs->u_empty[ur]);
                if (u < 0) break;
                const Unit U = decode(prm, u);
                for (int t = U.t_begin; t < U.t_end; ++t, ++i) {
                    const int xs = i % K::kXSlots, ys = i % kYSlots;
                    const int tbB = (2 * i) % K::kBufs, tbC = (2 * i + 1) % K::kBufs;
                    const uint32_t bcB = smem_u32(smem + K::kOffBC + tbB * K::kBCTile);
                    const uint32_t bcC = smem_u32(smem + K::kOffBC + tbC * K::kBCTile);
                    if (!wait_bar(&bs->tb_full[tbB], ((2 * i) / K::kBufs) & 1, bs, err)) goto drain;
                    if (!wait_bar(&bs->tb_full[tbC], ((2 * i + 1) / K::kBufs) & 1, bs, err)) goto drain;
                    // G = C B^T into the G/P' columns, free once the previous tile's masked
                    // product (factored) or its per-head masks (unfactored) are done
                    if (i > 0) {
                        if (prev_shared) {
                            if (!wait_bar(&bs->g_empty_mma, gm & 1, bs, err)) goto drain;
                            ++gm;
                        } else {
                            if (!wait_bar(&bs->g_empty_mask, gk & 1, bs, err)) goto drain;
                            ++gk;
                        }
                    }
                    tc_fence_after();
                    mma_state_dim_n<false, NS>(ksN, tmem + kColG, sw128_desc(bcC, 16, 1024), sw128_desc(bcB, 16, 1024), idG, 0u);
                    mma_commit(&bs->g_full);
                    const uint64_t dSA = sw128_desc(bcB, kAtom, 1024);
                    if (!wait_bar(&bs->wx_full[xs], (i / K::kXSlots) & 1, bs, err)) goto drain;
                    const bool shared = *(volatile int*)&bs->xmode[xs] != 0;
                    const uint64_t dX = sw128_desc(smem_u32(smem + K::kOffX + xs * K::kXBytes), kAtom, 1024);
                    if (shared) {
                        if (!wait_bar(&bs->s_empty, (i & 1) ^ 1, bs, err)) goto drain;
                        tc_fence_after();
#pragma unroll
                        for (int mh = 0; mh < K::kMH; ++mh)
                            mma_tokens_smem(tmem + kColS + 64 * mh, dSA + (uint64_t)((2 * mh * kAtom) >> 4), dX, idS);
                        mma_commit(&bs->s_full);
                        mma_commit(&bs->tb_empty[tbB]);    // this tile's B has served G and S
                        // the state term C (2^L h)^T onto Y'': its operand needs only the state
                        // entering the tile, so it goes ahead of the masked product
                        if (!issue_r(Pend{i, ys, tbC, true})) goto drain;
                        if (!wait_bar(&bs->p_full, psh & 1, bs, err)) goto drain;
                        ++psh;
                        tc_fence_after();
                        mma_tokens_tmem(tmem + kColY + 128 * ys, tmem + kColP, dX, idY);
                        mma_commit(&bs->x_empty[xs]);
                        mma_commit(&bs->g_empty_mma);
                        mma_commit(&bs->y_full[ys]);
                    } else {
                        // the rare form, out of line
                        if (!mma_unfactored_tile<NS>(bs, err, tmem, ys, xs, tbB, tbC, i, nsh, nrd, np, K::kMH, ksN, dX,
                                                 dSA, sw128_desc(smem_u32(smem + K::kOffBC + tbC * K::kBCTile), 16, 1024),
                                                 dH, idS, idY))
                            goto drain;
                        ++nsh;
                        ++nrd;
                    }
                    prev_shared = shared;
                }
            }
        drain:
            // every MMA issued so far is complete before TMEM is released
            mma_commit(&bs->fin);
            mbar_wait(&bs->fin, 0, 1u << 24);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ cumsum warp
        // Per tile: the dt of the pair's heads, the tile's form
        // (factored unless a head decays by more than 2^96 over it), and per head
        // the cumulative sum of dt A (log2 units) into a slot for the mask group.
        int m = 0, hi = 0;
        for (;; ++m) {
            const int ur = m % kURing;
            if (!__all_sync(0xffffffffu, wait_bar_idle(&bs->u_full[ur], (m / kURing) & 1, bs, err)))
                goto done;
            const int u = bs->uid[ur];
            mbar_arrive(&bs->u_empty[ur]);
            if (u < 0) break;
            const Unit U = decode(prm, u);
            for (int t = U.t_begin; t < U.t_end; ++t) {
                const int64_t t0 = (int64_t)t * kTile;
                // tokens past the sequence's end get dt = 0: they neither move the
                // state nor reach a stored row
                const int len = (int)min((int64_t)kTile, (int64_t)U.len - t0);
                const float* dtr = prm.dt + ((int64_t)U.b * T + U.tok0 + t0) * H + U.hb * np;
                float dtv[2][4];
#pragma unroll
                for (int e = 0; e < 2; ++e)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int tt = lane * 4 + q;
                        dtv[e][q] = (e < np && tt < len) ? __ldg(dtr + (int64_t)tt * H + e) : 0.f;
                    }
                float worst = 0.f;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    if (e >= np) break;
                    float sdt = dtv[e][0] + dtv[e][1] + dtv[e][2] + dtv[e][3];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) sdt += __shfl_xor_sync(0xffffffffu, sdt, off);
                    worst = fmaxf(worst, sdt * fabsf(__ldg(prm.A + U.hb * np + e)) * kLog2e);
                }
                const float mode = worst <= kSharedMaskRangeLog2 ? 1.f : 0.f;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    if (e >= np) break;
                    const int h = U.hb * np + e;
                    const float a2 = __ldg(prm.A + h) * kLog2e;
                    const float d_h = prm.D ? __ldg(prm.D + h) : 0.f;
                    const int c = hi % kCsSlots;
                    if (!__all_sync(0xffffffffu,
                                    wait_bar_idle(&bs->cs_empty[c], ((hi / kCsSlots) & 1) ^ 1, bs, err)))
                        goto done;
                    float run = 0.f, v[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        run += dtv[e][q] * a2;
                        v[q] = run;
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
                    reinterpret_cast<float4*>(cs)[lane] = make_float4(excl + v[0], excl + v[1], excl + v[2], excl + v[3]);
                    reinterpret_cast<float4*>(cs + kTile)[lane] = make_float4(dtv[e][0], dtv[e][1], dtv[e][2], dtv[e][3]);
                    if (lane == 0) {
                        cs[kCsL] = last;
                        cs[kCsD] = d_h;
                        cs[kCsMode] = mode;
                    }
                    __syncwarp();
                    mbar_arrive(&bs->cs_full[c]);
                    ++hi;
                }
            }
        }
    } else if (warp == 3) {
        // ------------------------------------------------------------ publisher
        // Per unit: once the chain group has stored the state leaving it, one fence
        // makes those stores visible GPU-wide and the flag of the next segment's unit
        // is released.
        if (lane == 0) {
            for (int m = 0;; ++m) {
                const int ur = m % kURing;
                if (!wait_bar_idle(&bs->u_full[ur], (m / kURing) & 1, bs, err)) goto done;
                const int u = bs->uid[ur];
                mbar_arrive(&bs->u_empty[ur]);
                if (u < 0) break;
                const Unit U = decode(prm, u);
                if (!wait_bar_idle(&bs->pub_full[m & 1], (m >> 1) & 1, bs, err)) goto done;
                if (prm.chained && U.s < prm.nseg - 1) {
                    fence_acq_rel_gpu();
                    st_release(prm.flags + flag_index(prm, U.b, U.s + 1, U.hb), 1);
                }
                mbar_arrive(&bs->pub_empty[m & 1]);
            }
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ mask group
        // Thread j owns token row j of the tile (its TMEM lane). Per tile and head:
        // the skip term D x_j / q_j (or D x_j) stored into the tile's Y'' accumulator
        // and w o x in place of the x tile (the B operand of S and of the factored
        // masked product); then P' = tril(C B^T) in place over G. An unfactored tile
        // first gets each head's P = G o exp(cs_j - cs_i) dt_i in the S slot and is
        // multiplied with the raw x tiles before they are scaled in place.
        const int wq = warp - 4;
        const int j = tid - 128;
        const int jj = j & 31;
        const uint32_t lb = (uint32_t)(wq * 32) << 16;
        int m = 0, i = 0, hi = 0, nsh = 0;
        for (;; ++m) {
            const int ur = m % kURing;
            if (!wait_bar_all(&bs->u_full[ur], (m / kURing) & 1, bs, err)) goto done;
            const int u = bs->uid[ur];
            mbar_arrive(&bs->u_empty[ur]);
            if (u < 0) break;
            const Unit U = decode(prm, u);
            for (int t = U.t_begin; t < U.t_end; ++t, ++i) {
                const int xs = i % K::kXSlots, ys = i % kYSlots;
                if (!wait_bar_all(&bs->cs_full[hi % kCsSlots], (hi / kCsSlots) & 1, bs, err)) goto done;
                const bool shared = cs_base[(hi % kCsSlots) * (kCsSlotBytes / 4) + kCsMode] != 0.f;
                if (!wait_bar_all(&bs->x_full[xs], (i / K::kXSlots) & 1, bs, err)) goto done;
                if (!wait_bar_all(&bs->y_empty[ys], ((i / kYSlots) & 1) ^ 1, bs, err)) goto done;
                float* yi = reinterpret_cast<float*>(smem + K::kOffYInfo + ys * kYInfoBytes);
                uint8_t* sxp = smem + K::kOffX + xs * K::kXBytes;
                if (!shared) {
                    // the rare form (a head decays by more than 2^96 over the tile): out of
                    // line, so that its registers and code stay off the common path
                    if (!mask_unfactored_tile(bs, err, cs_base, yi, sxp, tmem + lb, ys, xs, hi, np, i, nsh, j, wq))
                        goto done;
                    ++nsh;
                } else {
                    tc_fence_after();
                    __syncwarp();
                    for (int e = 0; e < np; ++e) {
                        const int c = (hi + e) % kCsSlots;
                        if (!wait_bar_all(&bs->cs_full[c], ((hi + e) / kCsSlots) & 1, bs, err)) goto done;
                        const float* cs = cs_base + c * (kCsSlotBytes / 4);
                        const float L = cs[kCsL], csj = cs[j];
                        const float up = ex2(L - csj);              // 2^(L - cs_j) <= 1
                        const float w = up * cs[kTile + j];         // w_j = 2^(L - cs_j) dt_j
                        const float dq = cs[kCsD] * up;             // D / q_j
                        // what the chain and epilogue groups need, kept with the tile's Y''
                        yi[e * kTile + j] = ex2(csj - L);           // q_j
                        if (j == 0) yi[kYiEL + e] = ex2(L);
                        uint8_t* sx = sxp + e * kAtom;
                        uint4 xv[8];
#pragma unroll
                        for (int c8 = 0; c8 < 8; ++c8) xv[c8] = *reinterpret_cast<const uint4*>(sx + swz(j, c8));
                        // skip term into head e's 64 columns of the tile's Y''
                        preload_skip(tmem + lb + kColY + 128 * ys + 64 * e, xv, dq);
                        const float2 w2 = make_float2(w, w);
#pragma unroll
                        for (int c8 = 0; c8 < 8; ++c8)
                            *reinterpret_cast<uint4*>(sx + swz(j, c8)) =
                                make_uint4(pack_bf16(mul2(w2, unpack_bf16(xv[c8].x))),
                                           pack_bf16(mul2(w2, unpack_bf16(xv[c8].y))),
                                           pack_bf16(mul2(w2, unpack_bf16(xv[c8].z))),
                                           pack_bf16(mul2(w2, unpack_bf16(xv[c8].w))));
                    }
                    if (j == 0) yi[kYiMode] = 1.f;
                    tmem_st_wait();
                    mbar_arrive(&bs->yi_full[ys]);
                    fence_proxy_async_smem();
                    if (j == 0) bs->xmode[xs] = 1;
                    tc_fence_before();
                    mbar_arrive(&bs->wx_full[xs]);
                    // P' = tril(G) in bf16 over G's first 64 columns: block blk reads G
                    // columns 32 blk.. and writes P' columns 16 blk.., both already read
                    if (!wait_bar_all(&bs->g_full, i & 1, bs, err)) goto done;
                    tc_fence_after();
                    __syncwarp();
#pragma unroll 1
                    for (int blk = 0; blk < 4; ++blk) {
                        uint32_t pk[16];
                        if (blk > wq) {
#pragma unroll
                            for (int q2 = 0; q2 < 16; ++q2) pk[q2] = 0u;
                        } else {
                            float gv[32];
                            tmem_ld32(tmem + lb + kColG + 32 * blk, gv);
                            tmem_ld_wait_regs(gv);
                            if (blk < wq) {
#pragma unroll
                                for (int q2 = 0; q2 < 16; ++q2) pk[q2] = pack_bf16(gv[2 * q2], gv[2 * q2 + 1]);
                            } else {
#pragma unroll
                                for (int q2 = 0; q2 < 16; ++q2)   // causal mask: column i kept while i <= row
                                    pk[q2] = pack_bf16(2 * q2 <= jj ? gv[2 * q2] : 0.f,
                                                       2 * q2 + 1 <= jj ? gv[2 * q2 + 1] : 0.f);
                            }
                        }
                        tmem_st16(tmem + lb + kColP + 16 * blk, pk);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(&bs->p_full);
                }
                for (int e = 0; e < np; ++e) mbar_arrive(&bs->cs_empty[(hi + e) % kCsSlots]);
                hi += np;
            }
        }
    } else if (warp >= 8 && warp < 16) {
        // ------------------------------------------------------------ chain group
        // Thread (q, lane) of warp 8 + 4 ph + q owns TMEM lane r = 32q + lane and head-dim
        // columns 32ph..32ph+31. The pair's state is V pieces of 32 values per thread,
        // carried in registers through the unit's tiles: piece v is head v of the pair
        // (state 128), or state rows r + 128 v of the one head (state 256); its S sits
        // at TMEM columns 64 v, its operand in atom v. Per tile: the operand of
        // C h^T (bf16 2^L h, or h), then h <- 2^L h + S. At the unit's end the state
        // goes to the next segment (or the final states).
        constexpr int V = K::kNP * K::kMH;   // 2
        const int q = warp & 3;
        const int ph = (warp - 8) >> 2;
        const int r = q * 32 + lane;
        const uint32_t lb = (uint32_t)(q * 32) << 16;
        const int N = prm.N;
        const int nv = np * K::kMH;
        float hv[V][32];
        auto load_entry = [&](const Unit& U) {
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const int e = v / K::kMH, mh = v % K::kMH;
                const int n = r + 128 * mh;
                const float* src = v < nv ? entry_src(prm, U, U.hb * np + e) : nullptr;
                if (src && n < N) {
                    const float* s0 = src + (int64_t)(32 * ph) * N + n;
#pragma unroll
                    for (int p2 = 0; p2 < 32; ++p2) hv[v][p2] = __ldcg(s0 + (int64_t)p2 * N);
                } else {
#pragma unroll
                    for (int p2 = 0; p2 < 32; ++p2) hv[v][p2] = 0.f;
                }
            }
        };
        int m = 0, i = 0;
        for (;; ++m) {
            const int ur = m % kURing;
            if (!wait_bar_all(&bs->u_full[ur], (m / kURing) & 1, bs, err)) goto done;
            const int u = bs->uid[ur];
            mbar_arrive(&bs->u_empty[ur]);
            if (u < 0) break;
            const Unit U = decode(prm, u);
            // The state entering the unit, loaded before its first tile is ready, so that
            // the loads overlap the mask group's work on that tile: a chained unit's
            // comes from the previous segment's unit once its flag is set (acquired by
            // one thread; the chain group's barrier orders the others' loads after it).
            // An empty document has no tiles: its final state is its initial state.
            if (prm.chained && U.s > 0) {
                const bool bad = tid == 256 && !acquire_entry_flag(prm, U, bs, err);
                if (named_bar_or(1, 256, bad)) goto done;
            }
            load_entry(U);
            for (int t = U.t_begin; t < U.t_end; ++t, ++i) {
                const int ys = i % kYSlots;
                if (!wait_bar_all(&bs->yi_full[ys], (i / kYSlots) & 1, bs, err)) goto done;
                const float* yi = reinterpret_cast<const float*>(smem + K::kOffYInfo + ys * kYInfoBytes);
                const bool shared = yi[kYiMode] != 0.f;
                // the operand of the tile's state term, from the state entering the tile:
                // 2^L h (factored) or h, once the previous tile's product has read it
                if (!wait_bar_all(&bs->h_free, (i & 1) ^ 1, bs, err)) goto done;
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    if (v >= nv) break;
                    const float sc = shared ? yi[kYiEL + v / K::kMH] : 1.f;
                    uint8_t* ha = smem + K::kOffH + v * kAtom;
#pragma unroll
                    for (int pc = 0; pc < 4; ++pc) {   // 8 head-dim columns at a time
                        uint32_t op[4];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2)
                            op[e2] = pack_bf16(sc * hv[v][8 * pc + 2 * e2], sc * hv[v][8 * pc + 2 * e2 + 1]);
                        *reinterpret_cast<uint4*>(ha + swz(r, 4 * ph + pc)) = make_uint4(op[0], op[1], op[2], op[3]);
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bs->h_full);
                // then the state leaving the tile: h <- 2^L h + S
                if (!wait_bar_all(&bs->s_full, i & 1, bs, err)) goto done;
                tc_fence_after();
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    if (v >= nv) break;
                    const float eL = yi[kYiEL + v / K::kMH];
#pragma unroll
                    for (int pc = 0; pc < 4; ++pc) {
                        float sv[8];
                        tmem_ld8(tmem + lb + kColS + 64 * v + 32 * ph + 8 * pc, sv);
                        tmem_ld_wait_regs(sv);
#pragma unroll
                        for (int e2 = 0; e2 < 8; ++e2) hv[v][8 * pc + e2] = fmaf(eL, hv[v][8 * pc + e2], sv[e2]);
                    }
                }
                tc_fence_before();
                mbar_arrive(shared ? &bs->s_empty : &bs->s_read);
            }
            // the state leaving the unit
            if (!wait_bar_all(&bs->pub_empty[m & 1], ((m >> 1) & 1) ^ 1, bs, err)) goto done;
#pragma unroll
            for (int v = 0; v < V; ++v) {
                if (v >= nv) break;
                const int e = v / K::kMH, mh = v % K::kMH;
                const int n = r + 128 * mh;
                float* dst = exit_dst(prm, U, U.hb * np + e);
                if (dst && n < N) {
                    float* d0 = dst + (int64_t)(32 * ph) * N + n;
#pragma unroll
                    for (int p2 = 0; p2 < 32; ++p2) __stcg(d0 + (int64_t)p2 * N, hv[v][p2]);
                }
            }
            mbar_arrive(&bs->pub_full[m & 1]);
        }
    } else if (warp >= 16) {
        // ------------------------------------------------------------ epilogue group
        // Thread (q, lane) of warp 16 + q owns token row r = 32q + lane (TMEM lane): per
        // tile and head y = q_r Y'' (or Y'' + 2^cs_r R) over all 64 columns, staged in
        // the warp's own 4 KB, then one TMA store of the warp's 32 rows.
        const int q = warp - 16;
        const int r = q * 32 + lane;
        const uint32_t lb = (uint32_t)(q * 32) << 16;
        uint8_t* stg = smem + K::kOffStage;
        int m = 0, i = 0;
        for (;; ++m) {
            const int ur = m % kURing;
            if (!wait_bar_all(&bs->u_full[ur], (m / kURing) & 1, bs, err)) goto done;
            const int u = bs->uid[ur];
            mbar_arrive(&bs->u_empty[ur]);
            if (u < 0) break;
            const Unit U = decode(prm, u);
            for (int t = U.t_begin; t < U.t_end; ++t, ++i) {
                const int ys = i % kYSlots;
                const int64_t t0 = (int64_t)t * kTile;
                if (!wait_bar_all(&bs->y_full[ys], (i / kYSlots) & 1, bs, err)) goto done;
                tc_fence_after();
                const float* yi = reinterpret_cast<const float*>(smem + K::kOffYInfo + ys * kYInfoBytes);
                const bool shared = yi[kYiMode] != 0.f;
                for (int e = 0; e < np; ++e) {
                    const float f = yi[e * kTile + r];
                    const float2 f2 = make_float2(f, f);
                    // the warp's previous store has read its staging rows
                    if (lane == 0) bulk_wait_group_read0();
                    __syncwarp();
                    if (shared) {
#pragma unroll 1
                        for (int pc = 0; pc < 4; ++pc) {
                            float yv[16];
                            tmem_ld16(tmem + lb + kColY + 128 * ys + 64 * e + 16 * pc, yv);
                            tmem_ld_wait_regs(yv);
#pragma unroll
                            for (int cc = 0; cc < 2; ++cc) {
                                uint32_t o[4];
#pragma unroll
                                for (int e2 = 0; e2 < 4; ++e2) {
                                    const int x0 = 8 * cc + 2 * e2;
                                    o[e2] = pack_bf16(mul2(f2, make_float2(yv[x0], yv[x0 + 1])));
                                }
                                *reinterpret_cast<uint4*>(stg + swz(r, 2 * pc + cc)) = make_uint4(o[0], o[1], o[2], o[3]);
                            }
                        }
                    } else {
                        stage_unfactored_row(tmem + lb, ys, e, f, stg, r);
                    }
                    if (e == np - 1) {
                        // the tile's accumulators are read: free them before the stores
                        tc_fence_before();
                        mbar_arrive(&bs->y_empty[ys]);
                        if (!shared) mbar_arrive_cnt(&bs->s_empty, 2);
                    }
                    const int hh = U.hb * np + e;
                    if (kGate && t0 + r < U.len)
                        gate_row(prm.z, prm.nw, prm.gs, prm.eps, stg, r, ((int64_t)U.b * T + U.tok0 + t0 + r) * H + hh, hh);
                    const int64_t row0 = t0 + 32 * q;   // the warp's first row in the sequence
                    if (row0 + 32 <= U.len) {
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_4d(&tm_y, stg + q * (kAtom / 4), 0, hh, (int)(U.tok0 + row0), U.b);
                            bulk_commit_group();
                        }
                    } else if (t0 + r < U.len) {
                        // the sequence ends inside the warp's rows: the rows after it belong to
                        // the next document (or lie past the row), so each thread stores its own
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(prm.y) +
                            (((int64_t)U.b * T + U.tok0 + t0 + r) * H + hh) * kP);
#pragma unroll
                        for (int c = 0; c < 8; ++c) dst[c] = *reinterpret_cast<const uint4*>(stg + swz(r, c));
                    }
                }
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

template <int NS, bool kGate>
cudaError_t launch_ns(const FusedLaunch& a, const Params& prm, cudaStream_t st) {
    using K = Cfg<NS>;
    auto kern = ssd_fused_kernel<NS, kGate>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)K::kSmem);
    if (e != cudaSuccess) return e;
    const int sms = num_sms();
    const int grid = prm.nunits < sms ? prm.nunits : sms;
    kern<<<grid, kThreads, K::kSmem, st>>>(a.maps[0], a.maps[1], a.maps[2], a.maps[3], prm);
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
    return (ns == 128 && (H / G) % 2 == 0) ? 2 : 1;
}

size_t fused_sync_ints(const Dims& d, int nseg) { return 2 + (size_t)(d.b * nseg * d.H); }

namespace {
constexpr int kVarlenSortMax = 8192;

// One thread per document: its rank among the documents ordered by decreasing
// length (ties: lower index first) places it in `order`, so that the longest
// documents' units are taken first and the last wave holds short ones.
__global__ void varlen_order_kernel(const int* __restrict__ cu, int ndoc, int64_t T, int sort,
                                    int* __restrict__ order, int* __restrict__ bad) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= ndoc) return;
    const int a = cu[k], e = cu[k + 1];
    if (a > e || a < 0 || (int64_t)e > T || (k == 0 && a != 0) || (k == ndoc - 1 && (int64_t)e != T))
        atomicExch(bad, 1);
    if (!sort) {
        order[k] = k;
        return;
    }
    const int len = e - a;
    int rank = 0;
    for (int j = 0; j < ndoc; ++j) {
        const int lj = __ldg(cu + j + 1) - __ldg(cu + j);
        rank += (lj > len) || (lj == len && j < k);
    }
    order[rank] = k;
}
}  // namespace

int varlen_sort_max() { return kVarlenSortMax; }

cudaError_t launch_varlen_order(const int* cu, int ndoc, int64_t T, int* order, int* bad,
                                cudaStream_t st) {
    if (ndoc <= 0) return cudaSuccess;
    varlen_order_kernel<<<(ndoc + 255) / 256, 256, 0, st>>>(cu, ndoc, T, ndoc <= kVarlenSortMax ? 1 : 0,
                                                            order, bad);
    return cudaGetLastError();
}

cudaError_t launch_fused(const FusedLaunch& a, cudaStream_t st) {
    const Dims& d = a.d;
    const int ns = fused_state_capacity(d.N);
    if (ns == 0 || a.nseg < 1 || a.seg_tiles < 1 || a.kheads < 1 || a.kheads > 2 || d.H % a.kheads != 0 ||
        (ns == 256 && a.kheads != 1))
        return cudaErrorInvalidValue;
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
    prm.y = a.y;
    prm.z = static_cast<const __nv_bfloat16*>(a.z);
    prm.nw = a.nw;
    prm.gs = a.gs;
    prm.eps = a.eps;
    if (a.z && (!a.nw || !fused_gate_ok(a.gs))) return cudaErrorInvalidValue;
    prm.cu = a.cu;
    prm.order = a.order;
    prm.T = d.T;
    prm.H = (int)d.H;
    prm.G = (int)d.G;
    prm.N = (int)d.N;
    prm.kheads = a.kheads;
    prm.batch = (int)d.b;
    const bool packed = a.cu != nullptr;
    if (!a.y || (packed && (!a.order || a.ndoc < 1 || d.b != 1 || a.nseg != 1 || a.chained)))
        return cudaErrorInvalidValue;
    // packed documents: every document's tiles start at tile 0, and at most all T
    // tokens form one document
    const int64_t ntiles = (d.T + kTile - 1) / kTile + (packed ? 1 : 0);
    const int64_t nunits = (packed ? (int64_t)a.ndoc : (int64_t)a.nseg * d.b) * (d.H / a.kheads);
    const int seg_first = a.seg_first > 0 ? a.seg_first : a.seg_tiles;
    if (nunits > INT32_MAX / 2 || d.T > INT32_MAX / 2 ||
        (!packed && seg_first + (int64_t)a.seg_tiles * (a.nseg - 1) < ntiles) || (!a.chained && seg_first != a.seg_tiles))
        return cudaErrorInvalidValue;
    prm.nunits = (int)nunits;
    prm.ntiles = (int)ntiles;
    prm.seg_tiles = a.seg_tiles;
    prm.seg_first = seg_first;
    prm.nseg = a.nseg;
    prm.nslot = a.nslot > 0 ? a.nslot : a.nseg;
    if (prm.nslot < a.nseg) return cudaErrorInvalidValue;
    prm.chained = a.chained;
    prm.stall = a.stall;
    if (a.z) return ns == 128 ? launch_ns<128, true>(a, prm, st) : launch_ns<256, true>(a, prm, st);
    return ns == 128 ? launch_ns<128, false>(a, prm, st) : launch_ns<256, false>(a, prm, st);
}

}  // namespace ssd
