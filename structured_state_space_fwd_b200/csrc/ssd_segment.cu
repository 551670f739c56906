// Segment states and the scan over segments, for long sequences ("Transformers
// are SSMs", Knowl 2: chunk states in parallel, then state passing across
// chunks; here the chunks are segments of several 128-token tiles).
//
// A sequence cut into segments of `seg_tiles` tiles is run by the single-pass
// kernel as one chain per segment, side by side, once the state entering every
// segment is known. These two kernels provide those states:
//
//   segment_state_kernel   per (segment s, batch row b, block of heads): the
//                          state the segment reaches from zero,
//                          S_s = sum_i 2^(E - cs_i) dt_i B_i x_i^T over its tokens
//                          (cs_i the inclusive cumulative sum of dt A from the
//                          segment start in log2 units, E its total), one long
//                          tcgen05 accumulation in tensor memory; and its decay 2^E.
//   segment_scan_kernel    h_0 = initial state, h_{s+1} = 2^E_s h_s + S_s, one
//                          thread per 4 state elements walking the segments.
//
// The weights 2^(E - cs_i) are relative to the segment's end, so they never
// exceed 1; contributions that underflow are below 2^-126 of the state.
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
constexpr int kThreads = 384;
constexpr uint32_t kAtom = kTile * 128;
constexpr int kMaxSegTiles = 64;
constexpr int kMaxHeads = 4;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

template <int NS>
struct SCfg {
    static constexpr int kMH = NS / 128;
    static constexpr uint32_t kBTile = (NS / 64) * kAtom;
    static constexpr int kBSlots = 2;
    static constexpr int kXSlots = NS == 128 ? 8 : 5;
    static constexpr int kAccBufs = NS == 128 ? 2 : 1;
    static constexpr uint32_t kOffB = 0;
    static constexpr uint32_t kOffX = kOffB + kBSlots * kBTile;
    static constexpr uint32_t kOffW = kOffX + kXSlots * kAtom;        // w per x slot
    static constexpr uint32_t kOffTot = kOffW + kXSlots * kTile * 4;  // tile totals [heads][tiles]
    static constexpr uint32_t kOffBar = kOffTot + 2 * kMaxHeads * kMaxSegTiles * 4;   // totals, suffix sums
    static constexpr uint32_t kSmem = kOffBar + 1024;
    static_assert(kSmem <= 232448, "shared memory budget");
    static_assert(kMaxHeads * 64 * kMH * kAccBufs <= 512, "tensor memory budget");
};

struct SParams {
    const float* dt;
    const float* A;
    float* segbuf;   // [b, nslot, H, P, N]
    float* decay;    // [b, nseg, H]
    int* error;
    int64_t T;
    int H, G, N, kheads, batch, seg_tiles, nseg, nslot, nunits, ntiles;
};

struct SBars {
    uint64_t b_full[2], b_empty[2];
    uint64_t x_full[8], x_empty[8], w_full[8], w_empty[8], wx_full[8];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t fin;
    uint32_t tmem;
    int abort;
};

__device__ __forceinline__ uint64_t gtime() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __noinline__ bool swait_slow(uint64_t* bar, uint32_t parity, SBars* bs, int* err) {
    const uint64_t t0 = gtime();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 15) == 0) {
            if (*(volatile int*)&bs->abort) return false;
            if (gtime() - t0 > kWaitLimitNs) {
                *(volatile int*)&bs->abort = 1;
                atomicExch(err, 3);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool swait(uint64_t* bar, uint32_t parity, SBars* bs, int* err) {
    if (mbar_try_wait(bar, parity)) return true;
    return swait_slow(bar, parity, bs, err);
}
__device__ __forceinline__ bool swait_all(uint64_t* bar, uint32_t parity, SBars* bs, int* err) {
    return __all_sync(0xffffffffu, swait(bar, parity, bs, err));
}
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack2(uint32_t u) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(h);
}

struct SUnit {
    int s, b, hb, t_begin, t_end;
};
__device__ __forceinline__ SUnit sdecode(const SParams& p, int u) {
    const int nhb = p.H / p.kheads;
    SUnit r;
    r.hb = u % nhb;
    r.b = (u / nhb) % p.batch;
    r.s = u / (nhb * p.batch);
    r.t_begin = r.s * p.seg_tiles;
    r.t_end = min(p.ntiles, r.t_begin + p.seg_tiles);
    return r;
}

// w o x in place for x tile nx (its slot's weights from the decay-weight warp),
// row j by this thread; false if a wait gave up.
template <int NS>
__device__ __forceinline__ bool scale_x_ns(uint8_t* smem, SBars* bs, int* err, int nx, int j) {
    using K = SCfg<NS>;
    const int xs = nx % K::kXSlots;
    if (!swait_all(&bs->x_full[xs], (nx / K::kXSlots) & 1, bs, err)) return false;
    if (!swait_all(&bs->w_full[xs], (nx / K::kXSlots) & 1, bs, err)) return false;
    const float w = reinterpret_cast<const float*>(smem + K::kOffW + xs * kTile * 4)[j];
    mbar_arrive(&bs->w_empty[xs]);
    const float2 w2 = make_float2(w, w);
    uint8_t* sx = smem + K::kOffX + xs * kAtom;
#pragma unroll
    for (int c8 = 0; c8 < 8; ++c8) {
        const uint32_t off = sw128_off(j, c8);
        const uint4 xv = *reinterpret_cast<const uint4*>(sx + off);
        float2 a = __fmul2_rn(w2, unpack2(xv.x)), b = __fmul2_rn(w2, unpack2(xv.y));
        float2 c = __fmul2_rn(w2, unpack2(xv.z)), d = __fmul2_rn(w2, unpack2(xv.w));
        *reinterpret_cast<uint4*>(sx + off) =
            make_uint4(pack2(a.x, a.y), pack2(b.x, b.y), pack2(c.x, c.y), pack2(d.x, d.y));
    }
    fence_proxy_async_smem();
    mbar_arrive(&bs->wx_full[xs]);
    return true;
}

template <int NS>
__global__ void __launch_bounds__(kThreads, 1)
    segment_state_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_B,
                         const SParams prm) {
    using K = SCfg<NS>;
    extern __shared__ __align__(1024) uint8_t smem[];
    SBars* bs = reinterpret_cast<SBars*>(smem + K::kOffBar);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int* err = prm.error;
    if (tid == 0) {
        if ((smem_u32(smem) & 1023u) != 0) atomicExch(err, 4);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bs->b_full[i], 1);
            mbar_init(&bs->b_empty[i], 1);
            mbar_init(&bs->acc_full[i], 1);
            mbar_init(&bs->acc_empty[i], 128);
        }
        for (int i = 0; i < 8; ++i) {
            mbar_init(&bs->x_full[i], 1);
            mbar_init(&bs->x_empty[i], 1);
            mbar_init(&bs->w_full[i], 32);
            mbar_init(&bs->w_empty[i], 128);
            mbar_init(&bs->wx_full[i], 128);
        }
        mbar_init(&bs->fin, 1);
        bs->abort = 0;
        fence_barrier_init();
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_B);
    }
    if (warp == 1) tmem_alloc(&bs->tmem, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const bool misaligned = (smem_u32(smem) & 1023u) != 0;
    const uint32_t tmem = bs->tmem;
    const int kh = prm.kheads;
    auto scale_x = [](uint8_t* sm, SBars* b, int* e, int n, int row) { return scale_x_ns<NS>(sm, b, e, n, row); };
    const int H = prm.H;
    const int64_t T = prm.T;
    const int natoms = (prm.N + 63) / 64;

    if (misaligned) {
    } else if (warp == 0) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            int nb = 0, nx = 0;
            for (int u = blockIdx.x; u < prm.nunits; u += gridDim.x) {
                const SUnit U = sdecode(prm, u);
                const int g = U.hb * kh / (H / prm.G);
                for (int t = U.t_begin; t < U.t_end; ++t, ++nb) {
                    const int sl = nb % K::kBSlots;
                    if (!swait(&bs->b_empty[sl], ((nb / K::kBSlots) & 1) ^ 1, bs, err)) goto pdrain;
                    mbar_arrive_expect_tx(&bs->b_full[sl], natoms * kAtom);
                    for (int a = 0; a < natoms; ++a)
                        tma_load_4d(smem + K::kOffB + sl * K::kBTile + a * kAtom, &tm_B, &bs->b_full[sl],
                                    a * 64, g, t * kTile, U.b);
                    for (int k = 0; k < kh; ++k, ++nx) {
                        const int xs = nx % K::kXSlots;
                        if (!swait(&bs->x_empty[xs], ((nx / K::kXSlots) & 1) ^ 1, bs, err)) {
                            ++nb;
                            goto pdrain;
                        }
                        mbar_arrive_expect_tx(&bs->x_full[xs], kAtom);
                        tma_load_4d(smem + K::kOffX + xs * kAtom, &tm_x, &bs->x_full[xs], 0, U.hb * kh + k,
                                    t * kTile, U.b);
                    }
                }
            }
        pdrain:
            for (int i = 0; i < K::kXSlots && i < nx; ++i)
                mbar_wait(&bs->x_full[(nx - 1 - i) % K::kXSlots], ((nx - 1 - i) / K::kXSlots) & 1, 1u << 22);
            for (int i = 0; i < K::kBSlots && i < nb; ++i)
                mbar_wait(&bs->b_full[(nb - 1 - i) % K::kBSlots], ((nb - 1 - i) / K::kBSlots) & 1, 1u << 22);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, kP, 1, 1);
            int nb = 0, nx = 0, nu = 0;
            for (int u = blockIdx.x; u < prm.nunits; u += gridDim.x, ++nu) {
                const SUnit U = sdecode(prm, u);
                const int ab = nu % K::kAccBufs;
                if (!swait(&bs->acc_empty[ab], ((nu / K::kAccBufs) & 1) ^ 1, bs, err)) goto drain;
                const uint32_t acc = tmem + (uint32_t)(ab * kMaxHeads * 64 * K::kMH);
                for (int t = U.t_begin; t < U.t_end; ++t, ++nb) {
                    const int sl = nb % K::kBSlots;
                    if (!swait(&bs->b_full[sl], (nb / K::kBSlots) & 1, bs, err)) goto drain;
                    const uint64_t dA = sw128_desc(smem_u32(smem + K::kOffB + sl * K::kBTile), kAtom, 1024);
                    for (int k = 0; k < kh; ++k, ++nx) {
                        const int xs = nx % K::kXSlots;
                        if (!swait(&bs->wx_full[xs], (nx / K::kXSlots) & 1, bs, err)) goto drain;
                        tc_fence_after();
                        const uint64_t dX = sw128_desc(smem_u32(smem + K::kOffX + xs * kAtom), kAtom, 1024);
                        for (int mh = 0; mh < K::kMH; ++mh)
                            for (int kk = 0; kk < kTile / 16; ++kk)
                                mma_bf16(acc + (uint32_t)((k * K::kMH + mh) * 64),
                                         dA + (uint64_t)((2 * mh * kAtom) >> 4) + (uint64_t)(kk * 128),
                                         dX + (uint64_t)(kk * 128), idS,
                                         (t > U.t_begin || kk > 0) ? 1u : 0u);
                        mma_commit(&bs->x_empty[xs]);
                    }
                    mma_commit(&bs->b_empty[sl]);
                }
                mma_commit(&bs->acc_full[ab]);
            }
        drain:
            mma_commit(&bs->fin);
            mbar_wait(&bs->fin, 0, 1u << 24);
        }
    } else if (warp == 2) {
        // ---------------------------------------------------------------- decay weights
        // Per unit and head: tile totals of dt A (log2 units), then per tile the
        // weights w_i = 2^(E - cs_i) dt_i with E - cs_i = (sum over later tiles)
        // + (tile total - inclusive sum to i), and the segment's decay 2^E.
        float* tot = reinterpret_cast<float*>(smem + K::kOffTot);
        int nx = 0;
        // dt of one tile for the unit's heads: lane l holds tokens 4l..4l+3; every load
        // of a tile is issued before any is used, so a tile costs one memory latency
        auto load_dt = [&](const SUnit& U, int tt, float (&dv)[kMaxHeads][4]) {
            const int64_t t0 = (int64_t)(U.t_begin + tt) * kTile + lane * 4;
#pragma unroll
            for (int k = 0; k < kMaxHeads; ++k)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dv[k][e] = (k < kh && t0 + e < T)
                                   ? __ldg(prm.dt + ((int64_t)U.b * T + t0 + e) * H + U.hb * kh + k)
                                   : 0.f;
        };
        for (int u = blockIdx.x; u < prm.nunits; u += gridDim.x) {
            const SUnit U = sdecode(prm, u);
            const int nt = U.t_end - U.t_begin;
            float a2[kMaxHeads];
#pragma unroll
            for (int k = 0; k < kMaxHeads; ++k) a2[k] = k < kh ? __ldg(prm.A + U.hb * kh + k) * kLog2e : 0.f;
            // tile totals of dt A per head, the next tile's dt loading during this one's sums
            float dv[kMaxHeads][4], dn[kMaxHeads][4];
            load_dt(U, 0, dv);
            for (int tt = 0; tt < nt; ++tt) {
                if (tt + 1 < nt) load_dt(U, tt + 1, dn);
#pragma unroll
                for (int k = 0; k < kMaxHeads; ++k) {
                    float sdt = dv[k][0] + dv[k][1] + dv[k][2] + dv[k][3];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) sdt += __shfl_xor_sync(0xffffffffu, sdt, off);
                    if (lane == 0 && k < kh) tot[k * kMaxSegTiles + tt] = sdt * a2[k];
                }
#pragma unroll
                for (int k = 0; k < kMaxHeads; ++k)
#pragma unroll
                    for (int e = 0; e < 4; ++e) dv[k][e] = dn[k][e];
            }
            __syncwarp();
            // suffix sums over later tiles, in place of the totals' copy kept per head:
            // lane k walks head k's tiles backwards; the segment's decay 2^E
            float* later = tot + kMaxHeads * kMaxSegTiles;
            if (lane < kh) {
                float acc = 0.f;
                for (int tt = nt - 1; tt >= 0; --tt) {
                    later[lane * kMaxSegTiles + tt] = acc;
                    acc += tot[lane * kMaxSegTiles + tt];
                }
                prm.decay[((int64_t)U.b * prm.nseg + U.s) * H + U.hb * kh + lane] = ex2(acc);
            }
            __syncwarp();
            load_dt(U, 0, dv);
            for (int tt = 0; tt < nt; ++tt) {
                if (tt + 1 < nt) load_dt(U, tt + 1, dn);
#pragma unroll
                for (int k = 0; k < kMaxHeads; ++k) {
                    if (k >= kh) break;
                    const float lat = later[k * kMaxSegTiles + tt];
                    const int xs = nx % K::kXSlots;
                    if (!swait_all(&bs->w_empty[xs], ((nx / K::kXSlots) & 1) ^ 1, bs, err)) goto done;
                    float run = 0.f, v[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        run += dv[k][e] * a2[k];
                        v[e] = run;
                    }
                    float incl = run;
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const float o = __shfl_up_sync(0xffffffffu, incl, off);
                        if (lane >= off) incl += o;
                    }
                    const float excl = incl - run;
                    const float ttot = __shfl_sync(0xffffffffu, incl, 31);
                    float* w = reinterpret_cast<float*>(smem + K::kOffW + xs * kTile * 4);
                    reinterpret_cast<float4*>(w)[lane] = make_float4(
                        ex2(lat + ttot - (excl + v[0])) * dv[k][0], ex2(lat + ttot - (excl + v[1])) * dv[k][1],
                        ex2(lat + ttot - (excl + v[2])) * dv[k][2], ex2(lat + ttot - (excl + v[3])) * dv[k][3]);
                    __syncwarp();
                    mbar_arrive(&bs->w_full[xs]);
                    ++nx;
                }
#pragma unroll
                for (int k = 0; k < kMaxHeads; ++k)
#pragma unroll
                    for (int e = 0; e < 4; ++e) dv[k][e] = dn[k][e];
            }
            __syncwarp();
        }
    } else if (warp >= 4 && warp < 8) {
        // ---------------------------------------------------------------- scale group
        // w o x in place for the even x tiles (the epilogue warps take the odd ones)
        const int j = tid - 128;
        int nx = 0;
        for (int u = blockIdx.x; u < prm.nunits; u += gridDim.x) {
            const SUnit U = sdecode(prm, u);
            for (int t = U.t_begin; t < U.t_end; ++t)
                for (int k = 0; k < kh; ++k, ++nx)
                    if (!(nx & 1) && !scale_x(smem, bs, err, nx, j)) goto done;
        }
    } else if (warp >= 8) {
        // ---------------------------------------------------------------- epilogue
        // thread (quarter q, lane) owns TMEM lane r: state row n = r (+128 per half)
        const int q = warp - 8;
        const int r = q * 32 + lane;
        const uint32_t lb = (uint32_t)(q * 32) << 16;
        const int N = prm.N;
        const int64_t PN = (int64_t)kP * N;
        int nu = 0, nx = 0;
        for (int u = blockIdx.x; u < prm.nunits; u += gridDim.x, ++nu) {
            const SUnit U = sdecode(prm, u);
            // first this unit's odd x tiles (every product of the unit needs them)
            for (int t = U.t_begin; t < U.t_end; ++t)
                for (int k = 0; k < kh; ++k, ++nx)
                    if ((nx & 1) && !scale_x(smem, bs, err, nx, r)) goto done;
            const int ab = nu % K::kAccBufs;
            if (!swait_all(&bs->acc_full[ab], (nu / K::kAccBufs) & 1, bs, err)) goto done;
            tc_fence_after();
            const uint32_t acc = tmem + (uint32_t)(ab * kMaxHeads * 64 * K::kMH);
            for (int k = 0; k < kh; ++k) {
                const int h = U.hb * kh + k;
                float* dst = prm.segbuf + (((int64_t)U.b * prm.nslot + U.s + 1) * H + h) * PN;
                for (int mh = 0; mh < K::kMH; ++mh) {
                    const int n = r + 128 * mh;
#pragma unroll 1
                    for (int hf = 0; hf < 2; ++hf) {
                        float v[32];
                        tmem_ld32(lb + acc + (uint32_t)((k * K::kMH + mh) * 64 + 32 * hf), v);
                        tmem_ld_wait_regs(v);
                        if (n < N) {
#pragma unroll
                            for (int p = 0; p < 32; ++p) dst[(int64_t)(32 * hf + p) * N + n] = v[p];
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bs->acc_empty[ab]);
        }
    }
done:
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// h_{s+1} = decay_s h_s + S_s over the segments, in place: slot s (s >= 1) holds
// S_{s-1} on entry and the state entering segment s on exit. With alpha_out, the
// thread of each (b, h)'s first vector also writes the product of the decays of
// segments 0 .. nseg_out - 1 there: the decay over all of them. The walk over the
// segments is a dependent chain of FMAs; the loads of the next kScanAhead slots are
// in flight while it runs. With store = 0 the slots are only read.
constexpr int kScanAhead = 8;
__global__ void segment_scan_kernel(const float* __restrict__ init, float* __restrict__ segbuf,
                                    const float* __restrict__ decay, int64_t nvec, int64_t H,
                                    int64_t PN4, int nseg, int nslot, int nseg_out, float* __restrict__ final_out,
                                    float* __restrict__ alpha_out, int store) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= nvec) return;
    const int64_t bh = e / PN4, off = e % PN4;
    const int64_t bi = bh / H, h = bh % H;
    float4 cur = init ? reinterpret_cast<const float4*>(init)[bh * PN4 + off] : make_float4(0.f, 0.f, 0.f, 0.f);
    float4* sb = reinterpret_cast<float4*>(segbuf);
    auto slot = [&](int s) { return ((bi * nslot + s) * H + h) * PN4 + off; };
    float4 ring[kScanAhead];
    float fr[kScanAhead];
#pragma unroll
    for (int k = 0; k < kScanAhead; ++k) {
        const int s = 1 + k;
        if (s <= nseg_out) {
            ring[k] = __ldcg(sb + slot(s));
            fr[k] = __ldg(decay + (bi * nseg + s - 1) * H + h);
        }
    }
    float prod = 1.f;
    for (int s0 = 1; s0 <= nseg_out; s0 += kScanAhead) {
#pragma unroll
        for (int k = 0; k < kScanAhead; ++k) {
            const int s = s0 + k;
            if (s > nseg_out) break;
            const float f = fr[k];
            const float4 v = ring[k];
            const int sn = s + kScanAhead;   // refill this ring entry with slot sn
            if (sn <= nseg_out) {
                ring[k] = __ldcg(sb + slot(sn));
                fr[k] = __ldg(decay + (bi * nseg + sn - 1) * H + h);
            }
            prod *= f;
            cur = make_float4(fmaf(f, cur.x, v.x), fmaf(f, cur.y, v.y), fmaf(f, cur.z, v.z), fmaf(f, cur.w, v.w));
            if (store && s < nslot) __stcg(sb + slot(s), cur);
        }
    }
    if (final_out) reinterpret_cast<float4*>(final_out)[bh * PN4 + off] = cur;
    if (alpha_out && off == 0) alpha_out[bh] = prod;
}

int sms_now() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

template <int NS>
cudaError_t launch_states_ns(const CUtensorMap* maps, const SParams& prm, cudaStream_t st) {
    using K = SCfg<NS>;
    cudaError_t e = cudaFuncSetAttribute(segment_state_kernel<NS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)K::kSmem);
    if (e != cudaSuccess) return e;
    const int sms = sms_now();
    const int grid = prm.nunits < sms ? prm.nunits : sms;
    segment_state_kernel<NS><<<grid, kThreads, K::kSmem, st>>>(maps[0], maps[1], prm);
    return cudaGetLastError();
}

}  // namespace

int segment_max_tiles() { return kMaxSegTiles; }

cudaError_t launch_segment_states(const Dims& d, const CUtensorMap* maps, const float* dt, const float* A,
                                  float* segbuf, float* decay, int* error, int seg_tiles, int nseg, int nslot,
                                  int nseg_out, int kheads, cudaStream_t st) {
    const int ns = fused_state_capacity(d.N);
    if (ns == 0 || seg_tiles < 1 || seg_tiles > kMaxSegTiles || kheads < 1 || kheads > kMaxHeads ||
        nseg_out < 0 || nseg_out > nseg || nslot < nseg_out + 1 || d.H % kheads != 0)
        return cudaErrorInvalidValue;
    if (nseg_out == 0 || d.b == 0) return cudaSuccess;
    SParams prm = {};
    prm.dt = dt;
    prm.A = A;
    prm.segbuf = segbuf;
    prm.decay = decay;
    prm.error = error;
    prm.T = d.T;
    prm.H = (int)d.H;
    prm.G = (int)d.G;
    prm.N = (int)d.N;
    prm.kheads = kheads;
    prm.batch = (int)d.b;
    prm.seg_tiles = seg_tiles;
    prm.nseg = nseg;
    prm.nslot = nslot;
    prm.ntiles = (int)((d.T + kTile - 1) / kTile);
    const int64_t nunits = (int64_t)nseg_out * d.b * (d.H / kheads);
    if (nunits > INT32_MAX) return cudaErrorInvalidValue;
    prm.nunits = (int)nunits;
    return ns == 128 ? launch_states_ns<128>(maps, prm, st) : launch_states_ns<256>(maps, prm, st);
}

cudaError_t launch_segment_scan(const Dims& d, const float* init, float* segbuf, const float* decay, int nseg,
                                int nslot, int nseg_out, float* final_out, cudaStream_t st, float* alpha_out,
                                bool store) {
    if ((d.P * d.N) % 4 != 0) return cudaErrorInvalidValue;
    const int64_t PN4 = d.P * d.N / 4;
    const int64_t nvec = d.b * d.H * PN4;
    if (nvec == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t blocks = (nvec + threads - 1) / threads;
    if (blocks > INT32_MAX) return cudaErrorInvalidValue;
    segment_scan_kernel<<<(unsigned)blocks, threads, 0, st>>>(init, segbuf, decay, nvec, d.H, PN4, nseg, nslot,
                                                              nseg_out, final_out, alpha_out, store ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace ssd
