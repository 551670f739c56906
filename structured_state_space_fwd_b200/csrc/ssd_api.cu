// C ABI of libssd: host-side argument checks, workspace layout and dispatch of
// the block-decomposition steps ("Transformers are SSMs", Knowl 2) onto the
// caller's stream. Nothing here allocates device memory or synchronizes,
// except ssd_fwd_host, whose contract is to return finished host outputs.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <vector>

#include "ssd.h"
#include "ssd_internal.h"

namespace {

thread_local char g_detail[256] = "";

void set_detail(const char* what, cudaError_t e) {
    snprintf(g_detail, sizeof(g_detail), "%s: %s (%d)", what, cudaGetErrorString(e), (int)e);
}

constexpr int64_t kMaxDim = 256;

bool is_pow2_chunk(int64_t q) {
    return q == 16 || q == 32 || q == 64 || q == 128 || q == 256;
}

// Shape rules shared by every entry point.
ssd_status_t check_shape(const ssd_shape_t* s) {
    if (!s) return SSD_ERR_INVALID_ARG;
    if (s->reserved != 0) return SSD_ERR_INVALID_ARG;
    if (s->batch < 0 || s->seqlen < 0) return SSD_ERR_INVALID_ARG;
    if (s->nheads < 1 || s->headdim < 1 || s->ngroups < 1 || s->dstate < 1)
        return SSD_ERR_INVALID_ARG;
    if (s->nheads % s->ngroups != 0) return SSD_ERR_INVALID_ARG;
    if (s->dtype != SSD_F32 && s->dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
    if (s->chunk_size < 1) return SSD_ERR_INVALID_ARG;
    if (!is_pow2_chunk(s->chunk_size)) return SSD_ERR_UNSUPPORTED;
    if (s->headdim > kMaxDim || s->dstate > kMaxDim) return SSD_ERR_UNSUPPORTED;
    // keep every element index well inside int64 and grid sizes inside CUDA limits
    const double tok = (double)s->batch * (double)s->seqlen;
    if (tok * (double)s->nheads * (double)s->headdim > 4.0e15) return SSD_ERR_UNSUPPORTED;
    if (tok * (double)s->ngroups * (double)s->dstate > 4.0e15) return SSD_ERR_UNSUPPORTED;
    if ((double)s->batch * s->nheads * s->headdim * s->dstate > 4.0e15) return SSD_ERR_UNSUPPORTED;
    if (s->batch > 65535) return SSD_ERR_UNSUPPORTED;                 // grid.z
    const int64_t nc = s->seqlen > 0 ? (s->seqlen + s->chunk_size - 1) / s->chunk_size : 0;
    if (nc * s->nheads > 2147483647LL) return SSD_ERR_UNSUPPORTED;    // grid.y
    if (s->nheads > 65535) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

size_t elem_size(int dtype) { return dtype == SSD_BF16 ? 2 : 4; }

struct Range {
    const void* p;
    size_t bytes;
};

bool overlaps(Range a, Range b) {
    if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0) return false;
    const uintptr_t a0 = (uintptr_t)a.p, b0 = (uintptr_t)b.p;
    return a0 < b0 + b.bytes && b0 < a0 + a.bytes;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

struct Sizes {
    size_t x, dt, hv, bc, st, cs, chunk_states;
};

Sizes sizes_of(const ssd::Dims& d) {
    Sizes z;
    const size_t es = elem_size(d.dtype);
    z.x = (size_t)(d.b * d.T * d.H * d.P) * es;
    z.dt = (size_t)(d.b * d.T * d.H) * 4;
    z.hv = (size_t)d.H * 4;
    z.bc = (size_t)(d.b * d.T * d.G * d.N) * es;
    z.st = (size_t)(d.b * d.H * d.P * d.N) * 4;
    z.cs = (size_t)(d.b * d.H * d.nc * d.Q) * 4;
    z.chunk_states = (size_t)(d.b * d.nc * d.H * d.P * d.N) * 4;
    return z;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Which kernels ssd_fwd runs. SSD_PATH (the library's one debug variable) forces a path for
// testing the paths against each other: "fused", "segmented", "steps" or "simt";
// a path the shape cannot take falls back to the next one down that list.
enum class Path { Fused, Segmented, Steps, Simt };

const char* path_override() { return getenv("SSD_PATH"); }

// The single-pass tensor-core kernel serves bf16 with head dim 64 and a state
// dim that is a multiple of 16 up to 256.
bool fused_ok(const ssd::Dims& d) {
    return d.dtype == SSD_BF16 && d.P == 64 && ssd::fused_state_capacity(d.N) != 0 &&
           d.T <= 0x7fffffffLL && ssd::tma_available();
}

// The single-pass kernel carries each (batch row, head pair) chain's state
// through a segment of tiles inside one CTA, and from segment to segment through
// a buffer and a flag. A chain's segments therefore run one after another; with
// few chains (batch rows x head pairs) and many tiles that sets the time, and the
// states entering all segments are computed first instead (segment states, a
// scan over them), so that every segment can run at once.
#ifndef SSD_CHAINED_MIN_CHAINS
#define SSD_CHAINED_MIN_CHAINS 112
#endif
#ifndef SSD_TARGET_UNITS
#define SSD_TARGET_UNITS (4 * 148)
#endif
constexpr int64_t kChainedMinChains = SSD_CHAINED_MIN_CHAINS;  // fewer chains: compute entering states first
constexpr int64_t kSegmentMinTiles = 8;
constexpr int64_t kTargetUnits = SSD_TARGET_UNITS;             // units wanted: about four waves of CTAs
#ifndef SSD_SEG_TARGET_UNITS
#define SSD_SEG_TARGET_UNITS (2 * 148)
#endif
// Segments whose entering states come from the segment-state pass and scan: fewer,
// longer ones (at most two waves), since every segment adds a state slot to both
// passes and a pipeline fill to each of its units.
constexpr int64_t kSegTargetUnits = SSD_SEG_TARGET_UNITS;
#ifndef SSD_CP_TARGET_UNITS
#define SSD_CP_TARGET_UNITS 148
#endif
// A context-parallel slice: its segment-state pass and scan run twice per rank step
// (record, then entering states), so fewer segments still (about one wave of the
// segment-state pass).
constexpr int64_t kCpTargetUnits = SSD_CP_TARGET_UNITS;
constexpr int64_t kSmCount = 148;
#ifndef SSD_FIRST_SEG_PCT
#define SSD_FIRST_SEG_PCT 75
#endif
constexpr int64_t kFirstSegPct = SSD_FIRST_SEG_PCT;   // two chained segments: the first's share of the tiles

int64_t fused_chains(const ssd::Dims& d) {
    const int ns = ssd::fused_state_capacity(d.N);
    return d.b * (d.H / ssd::fused_kheads(d.H, d.G, ns));
}

bool prefer_segments(const ssd::Dims& d) {
    const int64_t ntiles = (d.T + 127) / 128;
    return ntiles >= kSegmentMinTiles && fused_chains(d) < kChainedMinChains;
}

Path pick_path(const ssd::Dims& d) {
    const char* e = path_override();
    const bool fz = fused_ok(d);
    const bool tc = ssd::tc_supported(d);
    if (e && strcmp(e, "simt") == 0) return Path::Simt;
    if (e && strcmp(e, "steps") == 0) return tc ? Path::Steps : Path::Simt;
    if (e && strcmp(e, "fused") == 0) return fz ? Path::Fused : (tc ? Path::Steps : Path::Simt);
    if (e && strcmp(e, "segmented") == 0)
        return fz && d.T > 128 ? Path::Segmented : (fz ? Path::Fused : (tc ? Path::Steps : Path::Simt));
    if (fz) return prefer_segments(d) ? Path::Segmented : Path::Fused;
    return tc ? Path::Steps : Path::Simt;
}

bool steps_use_tc(const ssd::Dims& d) {
    const char* e = path_override();
    return !(e && strcmp(e, "simt") == 0) && ssd::tc_supported(d);
}

// How the single-pass kernel covers the sequence: heads per unit, tiles per
// segment (unit), segments; chained = entering states come from the previous
// segment's unit, otherwise from the segment-state pass and scan.
struct SegPlan {
    int kh, seg_tiles, nseg, seg_first;
    bool chained;
};
SegPlan seg_plan(const ssd::Dims& d, Path path) {
    SegPlan sp;
    const int ns = ssd::fused_state_capacity(d.N);
    sp.kh = ssd::fused_kheads(d.H, d.G, ns);
    sp.chained = path != Path::Segmented;
    const int64_t ntiles = d.T > 0 ? (d.T + 127) / 128 : 1;
    const int64_t chains = std::max<int64_t>(1, d.b * (d.H / sp.kh));
    // Chained segments of one chain run one after another, so with no more
    // chains than SMs splitting them only adds hand-offs to the critical path.
    // chained: at least kTargetUnits units; segmented: at most kSegTargetUnits, so
    // that the last of the two waves is not a third one of a few units
    int64_t nseg = sp.chained ? (kTargetUnits + chains - 1) / chains : kSegTargetUnits / chains;
    if (sp.chained && chains <= kSmCount) nseg = 1;
    if (path == Path::Segmented) nseg = std::max<int64_t>(2, nseg);
    nseg = std::max<int64_t>(1, std::min(nseg, ntiles));
    int64_t K = (ntiles + nseg - 1) / nseg;
    K = std::min<int64_t>(K, ssd::segment_max_tiles());
    sp.seg_tiles = (int)K;
    sp.nseg = (int)((ntiles + K - 1) / K);
    sp.seg_first = sp.seg_tiles;
    if (sp.chained && sp.nseg == 2) {
        // Two chained segments: the second ones, taken last, are the shorter, so that
        // the CTAs that take one more unit than others take a short one.
        const int64_t first = std::min<int64_t>(ntiles - 1, (ntiles * kFirstSegPct + 50) / 100);
        if (first > sp.seg_tiles) {
            sp.seg_first = (int)first;
            sp.seg_tiles = (int)(ntiles - first);
        }
    }
    return sp;
}

// Workspace of ssd_fwd, regions 256-byte aligned:
//   fused / segmented: [sync ints: ticket, error, flags[b*nseg*H] | segment states
//                       [b,nseg,H,P,N] (nseg > 1) | segment decays [b,nseg,H] (segmented)]
//   step paths:        [cs | chunk states S | entry states h_c]
struct FwdWorkspace {
    Path path;
    SegPlan sp;
    size_t off_cs, off_S, off_entry;        // step paths
    size_t off_sync, off_chain, off_seg, off_decay;  // single-pass paths
    size_t total;
};

FwdWorkspace fwd_workspace(const ssd::Dims& d) {
    const Sizes z = sizes_of(d);
    FwdWorkspace w = {};
    w.path = pick_path(d);
    if (w.path == Path::Fused || w.path == Path::Segmented) {
        w.sp = seg_plan(d, w.path);
        const size_t nseg = (size_t)w.sp.nseg;
        w.off_sync = 0;
        w.off_chain = align_up(sizeof(int) * ssd::fused_sync_ints(d, w.sp.nseg), 256);
        w.off_seg = w.off_chain;
        w.off_decay = w.off_seg + (nseg > 1 ? align_up(z.st * nseg, 256) : 0);
        w.total = w.off_decay + (nseg > 1 && !w.sp.chained ? align_up((size_t)(d.b * d.H) * nseg * 4, 256) : 0);
    } else {
        w.off_cs = 0;
        w.off_S = align_up(z.cs, 256);
        w.off_entry = w.off_S + align_up(z.chunk_states, 256);
        w.total = w.off_entry + align_up(z.chunk_states, 256);
    }
    if (d.b == 0 || d.T == 0) w.total = 0;
    return w;
}

ssd_status_t cuda_status(const char* what, cudaError_t e) {
    if (e == cudaSuccess) return SSD_OK;
    set_detail(what, e);
    return SSD_ERR_CUDA;
}

ssd_status_t check_fwd_args(const ssd_shape_t* shape, const void* x, const float* dt,
                            const float* A, const void* B, const void* C, const float* D,
                            const float* init, void* y, float* final_states,
                            const void* workspace, size_t workspace_bytes) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    const ssd::Dims d = ssd::make_dims(*shape);
    const Sizes z = sizes_of(d);
    // a pointer may be NULL only when its tensor has no elements
    if ((!x && z.x) || (!dt && z.dt) || !A || (!B && z.bc) || (!C && z.bc) || (!y && z.x))
        return SSD_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(y, 16))
        return SSD_ERR_INVALID_ARG;
    if (!aligned(dt, 4) || !aligned(A, 4) || (D && !aligned(D, 4))) return SSD_ERR_INVALID_ARG;
    if ((init && !aligned(init, 16)) || (final_states && !aligned(final_states, 16)))
        return SSD_ERR_INVALID_ARG;
    if (workspace && !aligned(workspace, 16)) return SSD_ERR_INVALID_ARG;
    const FwdWorkspace w = fwd_workspace(d);
    if (workspace_bytes < w.total || (w.total > 0 && !workspace)) return SSD_ERR_INVALID_ARG;
    const Range ins[] = {{x, z.x}, {dt, z.dt}, {A, z.hv}, {B, z.bc}, {C, z.bc},
                         {D, D ? z.hv : 0}, {init, init ? z.st : 0}};
    const Range outs[] = {{y, z.x}, {final_states, final_states ? z.st : 0},
                          {workspace, w.total}};
    for (const Range& o : outs) {
        for (const Range& i : ins)
            if (overlaps(o, i)) return SSD_ERR_INVALID_ARG;
    }
    for (int i = 0; i < 3; ++i)
        for (int j = i + 1; j < 3; ++j)
            if (overlaps(outs[i], outs[j])) return SSD_ERR_INVALID_ARG;
    if (final_states && init && final_states == init) return SSD_ERR_INVALID_ARG;
    return SSD_OK;
}

// test builds: SSD_TEST_STALL_CHAIN=1 makes every chain hand-off wait run out
int test_stall() {
#ifdef SSD_TEST_HOOKS
    const char* v = getenv("SSD_TEST_STALL_CHAIN");
    return (v && v[0] == '1') ? 1 : 0;
#else
    return 0;
#endif
}

// The gate and norm applied in the single-pass kernel's stores (z null: none).
struct FusedGate {
    const void* z = nullptr;
    const float* w = nullptr;
    int64_t group_size = 0;
    float eps = 0.f;
};

ssd_status_t run_fwd(const ssd::Dims& d, const void* x, const float* dt, const float* A,
                     const void* B, const void* C, const float* D, const float* init, void* y,
                     float* final_states, void* workspace, cudaStream_t stream,
                     const FusedGate& gate = FusedGate()) {
    if (d.b == 0) return SSD_OK;
    if (d.T == 0) return cuda_status("final states", ssd::launch_copy_or_zero_states(d, init, final_states, stream));
    const FwdWorkspace w = fwd_workspace(d);
    char* ws = (char*)workspace;
    ssd_status_t st;
    if (w.path == Path::Fused || w.path == Path::Segmented) {
        CUtensorMap maps[4];
        if (!ssd::make_tc_maps(d, x, B, C, y, maps)) {
            ssd::set_error_detail("tensor map encoding failed");
            return SSD_ERR_CUDA;
        }
        int* sync = (int*)(ws + w.off_sync);
        if ((st = cuda_status("sync area", cudaMemsetAsync(sync, 0, sizeof(int) * ssd::fused_sync_ints(d, w.sp.nseg),
                                                           stream))) != SSD_OK)
            return st;
        float* segbuf = w.sp.nseg > 1 ? (float*)(ws + w.off_seg) : nullptr;
        if (w.sp.nseg > 1 && !w.sp.chained) {
            float* decay = (float*)(ws + w.off_decay);
            if ((st = cuda_status("segment states",
                                  ssd::launch_segment_states(d, maps, dt, A, segbuf, decay, sync + 1, w.sp.seg_tiles,
                                                             w.sp.nseg, w.sp.nseg, w.sp.nseg - 1,
                                                             ssd::pick_kheads(d.H / d.G), stream))) != SSD_OK)
                return st;
            if ((st = cuda_status("segment scan", ssd::launch_segment_scan(d, init, segbuf, decay, w.sp.nseg, w.sp.nseg,
                                                                           w.sp.nseg - 1, nullptr, stream))) != SSD_OK)
                return st;
        }
        ssd::FusedLaunch a = {};
        a.d = d;
        a.maps = maps;
        a.dt = dt;
        a.A = A;
        a.D = D;
        a.init = init;
        a.finalbuf = final_states;
        a.segbuf = segbuf;
        a.sync_ints = sync;
        a.kheads = w.sp.kh;
        a.seg_tiles = w.sp.seg_tiles;
        a.seg_first = w.sp.seg_first;
        a.nseg = w.sp.nseg;
        a.chained = w.sp.chained ? 1 : 0;
        a.stall = test_stall();
        a.y = y;
        a.z = gate.z;
        a.nw = gate.w;
        a.gs = (int)gate.group_size;
        a.eps = gate.eps;
        return cuda_status("fused forward", ssd::launch_fused(a, stream));
    }
    float* cs = (float*)(ws + w.off_cs);
    float* S = (float*)(ws + w.off_S);
    float* entry = (float*)(ws + w.off_entry);
    const bool tc = w.path == Path::Steps;
    if ((st = cuda_status("chunk cumsum", ssd::launch_chunk_cumsum(d, dt, A, cs, stream))) != SSD_OK)
        return st;
    if ((st = cuda_status("chunk state",
                          tc ? ssd::launch_chunk_state_tc(d, x, dt, B, cs, S, stream)
                             : ssd::launch_chunk_state_simt(d, x, dt, B, cs, S, stream))) != SSD_OK)
        return st;
    if ((st = cuda_status("state passing", ssd::launch_state_passing(d, S, cs, init, entry,
                                                                      final_states, stream))) != SSD_OK)
        return st;
    return cuda_status("chunk scan",
                       tc ? ssd::launch_chunk_scan_tc(d, x, dt, B, C, D, cs, entry, y, stream)
                          : ssd::launch_chunk_scan_simt(d, x, dt, B, C, D, cs, entry, y, stream));
}

// The fused kernel's device status word (sync ints [1]) of the launch that last
// used this workspace: waits for `s`, then maps a nonzero word to SSD_ERR_TIMEOUT.
ssd_status_t read_device_status(const ssd::Dims& d, const void* workspace, cudaStream_t s) {
    const FwdWorkspace w = fwd_workspace(d);
    if ((w.path != Path::Fused && w.path != Path::Segmented) || w.total == 0 || d.b == 0 || d.T == 0)
        return SSD_OK;
    int word = 0;
    ssd_status_t st;
    const int* dev = (const int*)((const char*)workspace + w.off_sync) + 1;
    if ((st = cuda_status("status read", cudaMemcpyAsync(&word, dev, sizeof(int),
                                                         cudaMemcpyDeviceToHost, s))) != SSD_OK)
        return st;
    if ((st = cuda_status("stream synchronize", cudaStreamSynchronize(s))) != SSD_OK) return st;
    if (word == 0) return SSD_OK;
    snprintf(g_detail, sizeof(g_detail), "%s",
             word == 1   ? "fused kernel: a tile's entering state was not handed on in time (chain flag wait)"
             : word == 3 ? "fused kernel: an mbarrier wait between warp roles timed out"
             : word == 4 ? "fused kernel: shared memory base not 1024-byte aligned"
                         : "fused kernel: device error");
    return SSD_ERR_TIMEOUT;
}

// Sequence-parallel workspace. Shapes the single-pass kernel takes: ssd_cp_begin
// runs the segment-state pass over the slice and a scan that only reads it (the
// record is the state after the last segment and the product of the segment
// decays), and keeps A; ssd_cp_end folds the records into the entering state, scans
// the same segment states from it (the states entering every segment) and runs the
// single-pass kernel over the segments side by side:
//   [A | status words | segment states [b, nseg+1, H, P, N] | segment decays [b, nseg, H]
//    | entering state h_in | the kernel's ticket, status and flags].
// Other shapes (step paths; begin leaves cs and S for end):
//   [cs | chunk states S | entry states | entering state h_in].
// Regions are 256-byte aligned.
struct CpWorkspace {
    bool single_pass;
    int kh, seg_tiles, nseg;                  // single pass: the segment-state pass
    size_t off_sync, off_seg, off_decay;      // single pass, begin
    size_t off_A, off_fwd;                    // single pass: A kept by begin; the kernel's sync ints (end)
    size_t off_cs, off_S, off_entry, off_hin, total;
};
CpWorkspace cp_workspace(const ssd::Dims& d) {
    const Sizes z = sizes_of(d);
    CpWorkspace w = {};
    w.single_pass = fused_ok(d) && d.T > 0;
    if (w.single_pass) {
        const int64_t ntiles = (d.T + 127) / 128;
        w.kh = ssd::pick_kheads(d.H / d.G);
        const int64_t units_per_seg = std::max<int64_t>(1, d.b * (d.H / w.kh));
        int64_t nseg = std::max<int64_t>(1, std::min<int64_t>(ntiles, (kCpTargetUnits + units_per_seg - 1) / units_per_seg));
        int64_t K = std::min<int64_t>((ntiles + nseg - 1) / nseg, ssd::segment_max_tiles());
        w.seg_tiles = (int)K;
        w.nseg = (int)((ntiles + K - 1) / K);
        w.off_A = 0;
        w.off_sync = align_up(z.hv, 256);
        w.off_seg = w.off_sync + 256;
        w.off_decay = w.off_seg + align_up(z.st * (size_t)(w.nseg + 1), 256);
        w.off_hin = w.off_decay + align_up((size_t)(d.b * d.H * w.nseg) * 4, 256);
        w.off_fwd = w.off_hin + align_up(z.st, 256);
        w.total = w.off_fwd + align_up(sizeof(int) * ssd::fused_sync_ints(d, w.nseg), 256);
    } else {
        w.off_cs = 0;
        w.off_S = align_up(z.cs, 256);
        w.off_entry = w.off_S + align_up(z.chunk_states, 256);
        w.off_hin = w.off_entry + align_up(z.chunk_states, 256);
        w.total = w.off_hin + align_up(z.st, 256);
    }
    if (d.b == 0) w.total = 0;
    return w;
}
// The rank fold and the state copies run one thread per state element in a 1-D grid.
constexpr int64_t kMaxFlatStateElems = 256LL * 2147483647LL;

// One rank's record: its slice's state [b,H,P,N], then alpha [b,H], padded to 16 bytes.
size_t cp_record_floats(const ssd::Dims& d) {
    return align_up((size_t)(d.b * d.H * d.P * d.N + d.b * d.H), 4);
}

// ssd_fwd_host works through the batch in slices of rows so that the copies in,
// the forward and the copies out of different slices overlap (the two copy
// directions use separate copy engines). Each slice has its own forward
// workspace, so every slice's device status word survives until it is read.
constexpr int kHostMaxSlices = 8;
struct HostPlan {
    int64_t nslices, rows;     // slices of `rows` batch rows (the last may be shorter)
    size_t ws_slice;           // forward workspace of one full slice
};
HostPlan host_plan(const ssd::Dims& d) {
    HostPlan hp;
    hp.nslices = d.b < kHostMaxSlices ? (d.b > 0 ? d.b : 1) : kHostMaxSlices;
    // slices start at row boundaries: keep the 16-byte alignment of every tensor
    if (d.b > 0) {
        const Sizes z = sizes_of(d);
        for (size_t bytes : {z.x, z.dt, z.bc, z.st})
            if ((bytes / d.b) % 16 != 0) hp.nslices = 1;
    }
    hp.rows = d.b > 0 ? (d.b + hp.nslices - 1) / hp.nslices : 0;
    if (hp.rows > 0) hp.nslices = (d.b + hp.rows - 1) / hp.rows;
    ssd::Dims ds = d;
    ds.b = hp.rows;
    hp.ws_slice = align_up(fwd_workspace(ds).total, 256);
    return hp;
}


// The two copy streams and the events of one ssd_fwd_host call. Sets are kept
// per device in a pool and reused: a call takes one (creating it only when all
// are in use by concurrent calls) and returns it when done, so repeated calls
// create no CUDA objects. The pool lives until the process exits.
constexpr int kPoolDevices = 64;
struct HostCopySet {
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev[2 * kHostMaxSlices] = {};
};
std::mutex g_pool_mutex;
std::vector<HostCopySet*> g_pool[kPoolDevices];

void destroy_copy_set(HostCopySet* c) {
    for (cudaEvent_t e : c->ev)
        if (e) cudaEventDestroy(e);
    if (c->s_in) cudaStreamDestroy(c->s_in);
    if (c->s_out) cudaStreamDestroy(c->s_out);
    delete c;
}

// A copy set for device `dev` (the current one), or nullptr with the failing call's status in *st.
HostCopySet* take_copy_set(int dev, ssd_status_t* st) {
    {
        std::lock_guard<std::mutex> lock(g_pool_mutex);
        if (!g_pool[dev].empty()) {
            HostCopySet* c = g_pool[dev].back();
            g_pool[dev].pop_back();
            return c;
        }
    }
    HostCopySet* c = new HostCopySet;
    if ((*st = cuda_status("stream create", cudaStreamCreateWithFlags(&c->s_in, cudaStreamNonBlocking))) != SSD_OK ||
        (*st = cuda_status("stream create", cudaStreamCreateWithFlags(&c->s_out, cudaStreamNonBlocking))) != SSD_OK) {
        destroy_copy_set(c);
        return nullptr;
    }
    for (cudaEvent_t& e : c->ev)
        if ((*st = cuda_status("event create", cudaEventCreateWithFlags(&e, cudaEventDisableTiming))) != SSD_OK) {
            destroy_copy_set(c);
            return nullptr;
        }
    return c;
}

void return_copy_set(int dev, HostCopySet* c) {
    std::lock_guard<std::mutex> lock(g_pool_mutex);
    g_pool[dev].push_back(c);
}


// Packed documents: workspace [ticket, error, malformed-offsets flag, pad | order[ndoc]]
// on the single-pass kernel; [status words | one document's ssd_fwd workspace] for
// the shapes it does not take, which run document by document (step paths, whose
// workspace grows with the sequence, so the whole pack's bounds every document's).
constexpr size_t kVarlenSyncBytes = 256;
size_t varlen_workspace(const ssd::Dims& d, int64_t ndoc) {
    if (fused_ok(d)) return kVarlenSyncBytes + align_up((size_t)ndoc * 4, 256);
    return kVarlenSyncBytes + align_up(fwd_workspace(d).total, 256);
}

ssd_status_t check_varlen_shape(const ssd_shape_t* shape, int64_t ndoc) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (shape->batch != 1 || ndoc < 0 || (ndoc == 0 && shape->seqlen != 0)) return SSD_ERR_INVALID_ARG;
    if (ndoc > 1 << 24) return SSD_ERR_UNSUPPORTED;
    const ssd::Dims d = ssd::make_dims(*shape);
    if ((double)ndoc * (double)d.H > 1.0e9) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

// Packed documents on shapes the single-pass kernel does not take: the offsets are
// read back (the call waits for `s`), checked, and each document runs as its own
// forward on its slice of the pack, one after another on `s`.
ssd_status_t varlen_by_document(const ssd::Dims& d, const void* x, const float* dt, const float* A,
                                const void* B, const void* C, const float* D, const int32_t* cu,
                                int64_t ndoc, const float* init, void* y, float* final_states,
                                char* ws, cudaStream_t s) {
    std::vector<int32_t> h((size_t)ndoc + 1);
    ssd_status_t st;
    if ((st = cuda_status("cu_seqlens read", cudaMemcpyAsync(h.data(), cu, h.size() * 4, cudaMemcpyDeviceToHost,
                                                             s))) != SSD_OK ||
        (st = cuda_status("stream synchronize", cudaStreamSynchronize(s))) != SSD_OK)
        return st;
    if (h[0] != 0 || h[(size_t)ndoc] != d.T) goto bad;
    for (int64_t k = 0; k < ndoc; ++k)
        if (h[k + 1] < h[k]) goto bad;
    {
        const size_t es = elem_size(d.dtype);
        const size_t PN = (size_t)(d.H * d.P * d.N);
        for (int64_t k = 0; k < ndoc; ++k) {
            const int64_t a = h[k], len = h[k + 1] - h[k];
            ssd::Dims dk = d;
            dk.T = len;
            dk.nc = (len + d.Q - 1) / d.Q;
            const char* xk = (const char*)x + (size_t)(a * d.H * d.P) * es;
            const char* bk = (const char*)B + (size_t)(a * d.G * d.N) * es;
            const char* ck = (const char*)C + (size_t)(a * d.G * d.N) * es;
            char* yk = (char*)y + (size_t)(a * d.H * d.P) * es;
            if (len > 0 && (!aligned(xk, 16) || !aligned(bk, 16) || !aligned(ck, 16))) {
                ssd::set_error_detail("ssd_fwd_varlen: a document's slice of x, B or C does not start on "
                                      "16 bytes (H*P and G*N elements per token must allow it)");
                return SSD_ERR_INVALID_ARG;
            }
            if ((st = run_fwd(dk, xk, dt + a * d.H, A, bk, ck, D, init ? init + k * PN : nullptr, yk,
                              final_states ? final_states + k * PN : nullptr, ws, s)) != SSD_OK)
                return st;
        }
    }
    return SSD_OK;
bad:
    ssd::set_error_detail("ssd_fwd_varlen: cu_seqlens is not a non-decreasing list from 0 to seqlen");
    return SSD_ERR_INVALID_ARG;
}

}  // namespace

void ssd::set_error_detail(const char* msg) { snprintf(g_detail, sizeof(g_detail), "%s", msg); }

extern "C" {

const char* ssd_status_string(ssd_status_t s) {
    switch (s) {
        case SSD_OK: return "SSD_OK";
        case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG";
        case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED";
        case SSD_ERR_CUDA: return "SSD_ERR_CUDA";
        case SSD_ERR_TIMEOUT: return "SSD_ERR_TIMEOUT";
    }
    return "SSD_ERR_UNKNOWN";
}

const char* ssd_last_error_detail(void) { return g_detail; }

int ssd_version(void) { return 100; }

ssd_status_t ssd_fwd_plan(const ssd_shape_t* shape, const char** path, int* kernels) {
    if (!path || !kernels) return SSD_ERR_INVALID_ARG;
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    const ssd::Dims d = ssd::make_dims(*shape);
    const Path p = pick_path(d);
    *path = p == Path::Fused ? "fused" : p == Path::Segmented ? "segmented" : p == Path::Steps ? "steps" : "simt";
    *kernels = (d.b == 0) ? 0 : (d.T == 0 ? 1 : (p == Path::Fused ? 1 : p == Path::Segmented ? 3 : 4));
    return SSD_OK;
}

ssd_status_t ssd_fwd_workspace_size(const ssd_shape_t* shape, size_t* bytes) {
    if (!bytes) return SSD_ERR_INVALID_ARG;
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    *bytes = fwd_workspace(ssd::make_dims(*shape)).total;
    return SSD_OK;
}

ssd_status_t ssd_fwd(const ssd_shape_t* shape, const void* x, const float* dt, const float* A,
                     const void* B, const void* C, const float* D, const float* initial_states,
                     void* y, float* final_states, void* workspace, size_t workspace_bytes,
                     void* stream) {
    ssd_status_t st = check_fwd_args(shape, x, dt, A, B, C, D, initial_states, y, final_states,
                                     workspace, workspace_bytes);
    if (st != SSD_OK) return st;
    return run_fwd(ssd::make_dims(*shape), x, dt, A, B, C, D, initial_states, y, final_states,
                   workspace, (cudaStream_t)stream);
}

// Forward plus the gate and norm of the block: with `fuse`, the single-pass kernel
// applies them in its stores when the plan is single-pass and the groups lie inside
// a head; otherwise y goes to the workspace and the separate gate kernel follows.
bool gated_fuses(const ssd::Dims& d, int64_t group_size, int fuse) {
    const Path p = pick_path(d);
    return fuse && (p == Path::Fused || p == Path::Segmented) && ssd::fused_gate_ok(group_size);
}

ssd_status_t ssd_fwd_gated_workspace_size(const ssd_shape_t* shape, int64_t group_size, int fuse,
                                          size_t* bytes) {
    if (!bytes) return SSD_ERR_INVALID_ARG;
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    const ssd::Dims d = ssd::make_dims(*shape);
    if (group_size < 1 || (d.H * d.P) % group_size != 0) return SSD_ERR_INVALID_ARG;
    const size_t fw = fwd_workspace(d).total;
    *bytes = gated_fuses(d, group_size, fuse) ? fw : align_up(fw, 256) + sizes_of(d).x;
    return SSD_OK;
}

ssd_status_t ssd_fwd_gated(const ssd_shape_t* shape, const void* x, const float* dt, const float* A,
                           const void* B, const void* C, const float* D, const float* initial_states,
                           const void* z, const float* norm_weight, int64_t group_size, float eps,
                           int fuse, void* out, float* final_states, void* workspace,
                           size_t workspace_bytes, void* stream) {
    size_t need = 0;
    ssd_status_t st = ssd_fwd_gated_workspace_size(shape, group_size, fuse, &need);
    if (st != SSD_OK) return st;
    if (workspace_bytes < need || !(eps >= 0.f) || !std::isfinite(eps)) return SSD_ERR_INVALID_ARG;
    const ssd::Dims d = ssd::make_dims(*shape);
    const Sizes z0 = sizes_of(d);
    if ((!z && z0.x) || !norm_weight || !aligned(z, 16) || !aligned(norm_weight, 16)) return SSD_ERR_INVALID_ARG;
    const Range zr[] = {{z, z0.x}, {norm_weight, (size_t)(d.H * d.P) * 4}};
    for (const Range& r : zr)
        if (overlaps(r, Range{out, z0.x}) || overlaps(r, Range{final_states, final_states ? z0.st : 0}) ||
            overlaps(r, Range{workspace, need}))
            return SSD_ERR_INVALID_ARG;
    if (gated_fuses(d, group_size, fuse)) {
        // out takes y's place: every check of ssd_fwd applies to it
        if ((st = check_fwd_args(shape, x, dt, A, B, C, D, initial_states, out, final_states, workspace,
                                 workspace_bytes)) != SSD_OK)
            return st;
        FusedGate g;
        g.z = z;
        g.w = norm_weight;
        g.group_size = group_size;
        g.eps = eps;
        return run_fwd(d, x, dt, A, B, C, D, initial_states, out, final_states, workspace, (cudaStream_t)stream, g);
    }
    char* yb = (char*)workspace + align_up(fwd_workspace(d).total, 256);
    if ((st = check_fwd_args(shape, x, dt, A, B, C, D, initial_states, yb, final_states, workspace,
                             fwd_workspace(d).total)) != SSD_OK)
        return st;
    if (overlaps(Range{out, z0.x}, Range{workspace, need})) return SSD_ERR_INVALID_ARG;
    if ((st = run_fwd(d, x, dt, A, B, C, D, initial_states, yb, final_states, workspace,
                      (cudaStream_t)stream)) != SSD_OK)
        return st;
    return ssd_gated_rmsnorm(shape, yb, z, norm_weight, group_size, eps, out, stream);
}

// Host-buffer variant: [fwd workspace | x | dt | A | B | C | D | init | y | final]
ssd_status_t ssd_fwd_host_workspace_size(const ssd_shape_t* shape, size_t* bytes) {
    if (!bytes) return SSD_ERR_INVALID_ARG;
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    const ssd::Dims d = ssd::make_dims(*shape);
    const Sizes z = sizes_of(d);
    const HostPlan hp = host_plan(d);
    size_t tot = (size_t)hp.nslices * hp.ws_slice;
    for (size_t s : {z.x, z.dt, z.hv, z.bc, z.bc, z.hv, z.st, z.x, z.st}) tot += align_up(s, 256);
    *bytes = tot;
    return SSD_OK;
}

ssd_status_t ssd_fwd_host(const ssd_shape_t* shape, const void* x, const float* dt,
                          const float* A, const void* B, const void* C, const float* D,
                          const float* initial_states, void* y, float* final_states,
                          void* device_workspace, size_t workspace_bytes, void* stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    {
        const Sizes z0 = sizes_of(ssd::make_dims(*shape));
        if ((!x && z0.x) || (!dt && z0.dt) || !A || (!B && z0.bc) || (!C && z0.bc) || (!y && z0.x))
            return SSD_ERR_INVALID_ARG;
    }
    if (!device_workspace || !aligned(device_workspace, 256)) return SSD_ERR_INVALID_ARG;
    size_t need = 0;
    ssd_fwd_host_workspace_size(shape, &need);
    if (workspace_bytes < need) return SSD_ERR_INVALID_ARG;
    const ssd::Dims d = ssd::make_dims(*shape);
    const Sizes z = sizes_of(d);
    const HostPlan hp = host_plan(d);
    cudaStream_t s = (cudaStream_t)stream;
    char* base = (char*)device_workspace;
    size_t off = (size_t)hp.nslices * hp.ws_slice;
    auto take = [&](size_t bytes) {
        char* p = base + off;
        off += align_up(bytes, 256);
        return p;
    };
    char* dx = take(z.x);
    char* ddt = take(z.dt);
    float* dA = (float*)take(z.hv);
    char* dB = take(z.bc);
    char* dC = take(z.bc);
    float* dD = (float*)take(z.hv);
    char* dinit = take(z.st);
    char* dy = take(z.x);
    char* dfinal = take(z.st);
    if (d.b == 0) return SSD_OK;
    // bytes of one batch row of each batch-major tensor
    const size_t rx = z.x / d.b, rdt = z.dt / d.b, rbc = z.bc / d.b, rst = z.st / d.b;
    int dev = -1;
    if ((st = cuda_status("current device", cudaGetDevice(&dev))) != SSD_OK) return st;
    if (dev < 0 || dev >= kPoolDevices) {
        ssd::set_error_detail("ssd_fwd_host: device ordinal beyond the copy-stream pool");
        return SSD_ERR_UNSUPPORTED;
    }
    HostCopySet* cs = take_copy_set(dev, &st);
    if (!cs) return st;
    cudaStream_t s_in = cs->s_in, s_out = cs->s_out;
    cudaEvent_t* ev = cs->ev;
    // every way out waits for the call's copies and kernels, then returns the set
    auto fail = [&](ssd_status_t r) {
        cudaStreamSynchronize(s);
        cudaStreamSynchronize(s_in);
        cudaStreamSynchronize(s_out);
        return_copy_set(dev, cs);
        return r;
    };
    // s_in starts after whatever the caller queued on `stream` before this call
    if ((st = cuda_status("event record", cudaEventRecord(ev[0], s))) != SSD_OK ||
        (st = cuda_status("stream wait", cudaStreamWaitEvent(s_in, ev[0], 0))) != SSD_OK)
        return fail(st);
    auto h2d = [&](void* dst, const void* src, size_t n) -> ssd_status_t {
        if (n == 0) return SSD_OK;
        return cuda_status("host to device copy", cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, s_in));
    };
    auto d2h = [&](void* dst, const void* src, size_t n) -> ssd_status_t {
        if (n == 0) return SSD_OK;
        return cuda_status("device to host copy", cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToHost, s_out));
    };
    if ((st = h2d(dA, A, z.hv)) != SSD_OK || (st = h2d(dD, D, D ? z.hv : 0)) != SSD_OK) return fail(st);
    for (int64_t k = 0; k < hp.nslices; ++k) {
        const int64_t r0 = k * hp.rows, nr = std::min(hp.rows, d.b - r0);
        ssd::Dims ds = d;
        ds.b = nr;
        if ((st = h2d(dx + r0 * rx, (const char*)x + r0 * rx, nr * rx)) != SSD_OK ||
            (st = h2d(ddt + r0 * rdt, (const char*)dt + r0 * rdt, nr * rdt)) != SSD_OK ||
            (st = h2d(dB + r0 * rbc, (const char*)B + r0 * rbc, nr * rbc)) != SSD_OK ||
            (st = h2d(dC + r0 * rbc, (const char*)C + r0 * rbc, nr * rbc)) != SSD_OK ||
            (st = h2d(dinit + r0 * rst, initial_states ? (const char*)initial_states + r0 * rst : nullptr,
                      initial_states ? nr * rst : 0)) != SSD_OK)
            return fail(st);
        if ((st = cuda_status("event record", cudaEventRecord(ev[2 * k], s_in))) != SSD_OK ||
            (st = cuda_status("stream wait", cudaStreamWaitEvent(s, ev[2 * k], 0))) != SSD_OK)
            return fail(st);
        st = run_fwd(ds, dx + r0 * rx, (const float*)(ddt + r0 * rdt), dA, dB + r0 * rbc, dC + r0 * rbc,
                     D ? dD : nullptr, initial_states ? (const float*)(dinit + r0 * rst) : nullptr,
                     dy + r0 * rx, final_states ? (float*)(dfinal + r0 * rst) : nullptr,
                     base + (size_t)k * hp.ws_slice, s);
        if (st != SSD_OK) return fail(st);
        if ((st = cuda_status("event record", cudaEventRecord(ev[2 * k + 1], s))) != SSD_OK ||
            (st = cuda_status("stream wait", cudaStreamWaitEvent(s_out, ev[2 * k + 1], 0))) != SSD_OK)
            return fail(st);
        if ((st = d2h((char*)y + r0 * rx, dy + r0 * rx, nr * rx)) != SSD_OK ||
            (st = d2h(final_states ? (char*)final_states + r0 * rst : nullptr, dfinal + r0 * rst,
                      final_states ? nr * rst : 0)) != SSD_OK)
            return fail(st);
    }
    if ((st = cuda_status("stream synchronize", cudaStreamSynchronize(s_out))) != SSD_OK ||
        (st = cuda_status("stream synchronize", cudaStreamSynchronize(s))) != SSD_OK)
        return fail(st);
    return_copy_set(dev, cs);
    // every slice's fused kernel reports through its own status word
    for (int64_t k = 0; k < hp.nslices; ++k) {
        ssd::Dims ds = d;
        ds.b = std::min(hp.rows, d.b - k * hp.rows);
        if ((st = read_device_status(ds, base + (size_t)k * hp.ws_slice, s)) != SSD_OK) return st;
    }
    return SSD_OK;
}

ssd_status_t ssd_fwd_check(const ssd_shape_t* shape, const void* workspace, size_t workspace_bytes,
                           void* stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    const ssd::Dims d = ssd::make_dims(*shape);
    const FwdWorkspace w = fwd_workspace(d);
    if (workspace_bytes < w.total || (w.total > 0 && !workspace)) return SSD_ERR_INVALID_ARG;
    return read_device_status(d, workspace, (cudaStream_t)stream);
}

ssd_status_t ssd_fwd_varlen_workspace_size(const ssd_shape_t* shape, int64_t n_docs, size_t* bytes) {
    if (!bytes) return SSD_ERR_INVALID_ARG;
    ssd_status_t st = check_varlen_shape(shape, n_docs);
    if (st != SSD_OK) return st;
    *bytes = n_docs > 0 ? varlen_workspace(ssd::make_dims(*shape), n_docs) : 0;
    return SSD_OK;
}

ssd_status_t ssd_fwd_varlen(const ssd_shape_t* shape, const void* x, const float* dt, const float* A,
                            const void* B, const void* C, const float* D, const int32_t* cu_seqlens,
                            int64_t n_docs, const float* initial_states, void* y, float* final_states,
                            void* workspace, size_t workspace_bytes, void* stream) {
    ssd_status_t st = check_varlen_shape(shape, n_docs);
    if (st != SSD_OK) return st;
    if (n_docs == 0) return SSD_OK;
    const ssd::Dims d = ssd::make_dims(*shape);
    const Sizes z = sizes_of(d);
    const size_t zst = (size_t)(n_docs * d.H * d.P * d.N) * 4;    // [n_docs,H,P,N] states
    const size_t need = varlen_workspace(d, n_docs);
    if ((!x && z.x) || (!dt && z.dt) || !A || (!B && z.bc) || (!C && z.bc) || (!y && z.x) || !cu_seqlens ||
        !workspace)
        return SSD_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(y, 16) || !aligned(workspace, 16))
        return SSD_ERR_INVALID_ARG;
    if (!aligned(dt, 4) || !aligned(A, 4) || (D && !aligned(D, 4)) || !aligned(cu_seqlens, 4))
        return SSD_ERR_INVALID_ARG;
    if ((initial_states && !aligned(initial_states, 16)) || (final_states && !aligned(final_states, 16)))
        return SSD_ERR_INVALID_ARG;
    if (workspace_bytes < need) return SSD_ERR_INVALID_ARG;
    const Range ins[] = {{x, z.x}, {dt, z.dt}, {A, z.hv}, {B, z.bc}, {C, z.bc}, {D, D ? z.hv : 0},
                         {initial_states, initial_states ? zst : 0}, {cu_seqlens, (size_t)(n_docs + 1) * 4}};
    const Range outs[] = {{y, z.x}, {final_states, final_states ? zst : 0}, {workspace, need}};
    for (const Range& o : outs)
        for (const Range& i : ins)
            if (overlaps(o, i)) return SSD_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i)
        for (int j = i + 1; j < 3; ++j)
            if (overlaps(outs[i], outs[j])) return SSD_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    int* sync = (int*)ws;
    int* order = (int*)(ws + kVarlenSyncBytes);
    if ((st = cuda_status("sync area", cudaMemsetAsync(sync, 0, 16, s))) != SSD_OK) return st;
    if (!fused_ok(d))
        return varlen_by_document(d, x, dt, A, B, C, D, cu_seqlens, n_docs, initial_states, y, final_states,
                                  ws + kVarlenSyncBytes, s);
    if ((st = cuda_status("document order", ssd::launch_varlen_order(cu_seqlens, (int)n_docs, d.T, order,
                                                                      sync + 2, s))) != SSD_OK)
        return st;
    if (d.T == 0) {   // every document is empty: final states are the initial ones
        ssd::Dims dd = d;
        dd.b = n_docs;
        return cuda_status("final states", ssd::launch_copy_or_zero_states(dd, initial_states, final_states, s));
    }
    CUtensorMap maps[4];
    if (!ssd::make_tc_maps(d, x, B, C, y, maps)) {
        ssd::set_error_detail("tensor map encoding failed");
        return SSD_ERR_CUDA;
    }
    ssd::FusedLaunch a = {};
    a.d = d;
    a.maps = maps;
    a.dt = dt;
    a.A = A;
    a.D = D;
    a.init = initial_states;
    a.finalbuf = final_states;
    a.segbuf = nullptr;
    a.sync_ints = sync;
    a.kheads = ssd::fused_kheads(d.H, d.G, ssd::fused_state_capacity(d.N));
    a.seg_tiles = 1;
    a.nseg = 1;
    a.chained = 0;
    a.stall = 0;
    a.y = y;
    a.cu = cu_seqlens;
    a.order = order;
    a.ndoc = (int)n_docs;
    return cuda_status("fused forward (packed documents)", ssd::launch_fused(a, s));
}

ssd_status_t ssd_fwd_varlen_check(const ssd_shape_t* shape, int64_t n_docs, const void* workspace,
                                  size_t workspace_bytes, void* stream) {
    ssd_status_t st = check_varlen_shape(shape, n_docs);
    if (st != SSD_OK) return st;
    if (n_docs == 0) return SSD_OK;
    if (!workspace || workspace_bytes < varlen_workspace(ssd::make_dims(*shape), n_docs))
        return SSD_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    int words[3] = {0, 0, 0};
    if ((st = cuda_status("status read", cudaMemcpyAsync(words, workspace, sizeof(words),
                                                         cudaMemcpyDeviceToHost, s))) != SSD_OK)
        return st;
    if ((st = cuda_status("stream synchronize", cudaStreamSynchronize(s))) != SSD_OK) return st;
    if (words[2] != 0) {
        ssd::set_error_detail("ssd_fwd_varlen: cu_seqlens is not a non-decreasing list from 0 to seqlen "
                              "(offsets were clamped into the row; outputs are not meaningful)");
        return SSD_ERR_INVALID_ARG;
    }
    if (words[1] != 0) {
        ssd::set_error_detail(words[1] == 3 ? "fused kernel: an mbarrier wait between warp roles timed out"
                                            : "fused kernel: device error");
        return SSD_ERR_TIMEOUT;
    }
    return SSD_OK;
}

ssd_status_t ssd_step(const ssd_shape_t* shape, const void* x, const float* dt, const float* A,
                      const void* B, const void* C, const float* D, float* state, void* y,
                      void* stream) {
    if (!shape) return SSD_ERR_INVALID_ARG;
    ssd_shape_t s = *shape;
    s.chunk_size = 64;   // not used by the recurrent form
    ssd_status_t st = check_shape(&s);
    if (st != SSD_OK) return st;
    const ssd::Dims d = ssd::make_dims(s);
    const Sizes z = sizes_of(d);
    if ((!x && z.x) || (!dt && z.dt) || !A || (!B && z.bc) || (!C && z.bc) || (!y && z.x) ||
        (!state && z.st))
        return SSD_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(y, 16) || !aligned(state, 16))
        return SSD_ERR_INVALID_ARG;
    if (!aligned(dt, 4) || !aligned(A, 4) || (D && !aligned(D, 4))) return SSD_ERR_INVALID_ARG;
    const Range ins[] = {{x, z.x}, {dt, z.dt}, {A, z.hv}, {B, z.bc}, {C, z.bc}, {D, D ? z.hv : 0}};
    const Range outs[] = {{state, z.st}, {y, z.x}};
    for (const Range& o : outs)
        for (const Range& i : ins)
            if (overlaps(o, i)) return SSD_ERR_INVALID_ARG;
    if (overlaps(outs[0], outs[1])) return SSD_ERR_INVALID_ARG;
    return cuda_status("recurrent step", ssd::launch_step(d, x, dt, A, B, C, D, state, y,
                                                          (cudaStream_t)stream));
}

ssd_status_t ssd_cp_record_floats(const ssd_shape_t* shape, size_t* floats) {
    if (!floats) return SSD_ERR_INVALID_ARG;
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    *floats = cp_record_floats(ssd::make_dims(*shape));
    return SSD_OK;
}

ssd_status_t ssd_cp_workspace_size(const ssd_shape_t* shape, size_t* bytes) {
    if (!bytes) return SSD_ERR_INVALID_ARG;
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    *bytes = cp_workspace(ssd::make_dims(*shape)).total;
    return SSD_OK;
}

ssd_status_t ssd_cp_begin(const ssd_shape_t* shape, const void* x, const float* dt, const float* A,
                          const void* B, const float* initial_states, float* record,
                          void* workspace, size_t workspace_bytes, void* stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    const ssd::Dims d = ssd::make_dims(*shape);
    const Sizes z = sizes_of(d);
    const size_t rec_bytes = cp_record_floats(d) * 4;
    const CpWorkspace w = cp_workspace(d);
    if ((!x && z.x) || (!dt && z.dt) || !A || (!B && z.bc) || (!record && rec_bytes))
        return SSD_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(record, 16) || !aligned(workspace, 16) ||
        (initial_states && !aligned(initial_states, 16)) || !aligned(dt, 4) || !aligned(A, 4))
        return SSD_ERR_INVALID_ARG;
    if (workspace_bytes < w.total || (w.total > 0 && !workspace)) return SSD_ERR_INVALID_ARG;
    const Range ins[] = {{x, z.x}, {dt, z.dt}, {A, z.hv}, {B, z.bc},
                         {initial_states, initial_states ? z.st : 0}};
    const Range outs[] = {{record, rec_bytes}, {workspace, w.total}};
    for (const Range& o : outs)
        for (const Range& i : ins)
            if (overlaps(o, i)) return SSD_ERR_INVALID_ARG;
    if (overlaps(outs[0], outs[1])) return SSD_ERR_INVALID_ARG;
    if (d.b * d.H * d.P * d.N > kMaxFlatStateElems) return SSD_ERR_UNSUPPORTED;
    if (d.b == 0) return SSD_OK;
    cudaStream_t s = (cudaStream_t)stream;
    float* alpha = record + d.b * d.H * d.P * d.N;
    if (d.T == 0) {
        if ((st = cuda_status("slice state", ssd::launch_copy_or_zero_states(d, initial_states, record, s))) != SSD_OK)
            return st;
        return cuda_status("slice decay", ssd::launch_slice_decay(d, nullptr, alpha, s));
    }
    char* ws = (char*)workspace;
    if (w.single_pass) {
        CUtensorMap maps[4];
        if (!ssd::make_tc_maps(d, x, B, B, nullptr, maps)) {
            ssd::set_error_detail("tensor map encoding failed");
            return SSD_ERR_CUDA;
        }
        int* sync = (int*)(ws + w.off_sync);
        float* segbuf = (float*)(ws + w.off_seg);
        float* decay = (float*)(ws + w.off_decay);
        const int nslot = w.nseg + 1;
        if ((st = cuda_status("status word", cudaMemsetAsync(sync, 0, 16, s))) != SSD_OK ||
            (st = cuda_status("A for the slice's forward", cudaMemcpyAsync(ws + w.off_A, A, z.hv,
                                                                           cudaMemcpyDeviceToDevice, s))) != SSD_OK)
            return st;
        if ((st = cuda_status("segment states",
                              ssd::launch_segment_states(d, maps, dt, A, segbuf, decay, sync + 1, w.seg_tiles,
                                                         w.nseg, nslot, w.nseg, w.kh, s))) != SSD_OK)
            return st;
        // the slots keep the states from zero: ssd_cp_end scans them again from h_in
        return cuda_status("segment scan", ssd::launch_segment_scan(d, initial_states, segbuf, decay, w.nseg,
                                                                    nslot, w.nseg, record, s, alpha, false));
    }
    float* cs = (float*)(ws + w.off_cs);
    float* S = (float*)(ws + w.off_S);
    if ((st = cuda_status("chunk cumsum", ssd::launch_chunk_cumsum(d, dt, A, cs, s))) != SSD_OK) return st;
    if ((st = cuda_status("chunk state",
                          steps_use_tc(d) ? ssd::launch_chunk_state_tc(d, x, dt, B, cs, S, s)
                                          : ssd::launch_chunk_state_simt(d, x, dt, B, cs, S, s))) != SSD_OK)
        return st;
    if ((st = cuda_status("slice state", ssd::launch_state_passing(d, S, cs, initial_states, nullptr,
                                                                    record, s))) != SSD_OK)
        return st;
    return cuda_status("slice decay", ssd::launch_slice_decay(d, cs, alpha, s));
}

ssd_status_t ssd_cp_end(const ssd_shape_t* shape, int nranks, int rank, const float* records,
                        const float* initial_states, const void* x, const float* dt,
                        const void* B, const void* C, const float* D, void* y,
                        float* final_states, void* workspace, size_t workspace_bytes,
                        void* stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (nranks < 1 || rank < 0 || rank >= nranks) return SSD_ERR_INVALID_ARG;
    const ssd::Dims d = ssd::make_dims(*shape);
    const Sizes z = sizes_of(d);
    const size_t rec_floats = cp_record_floats(d);
    const size_t recs_bytes = rec_floats * 4 * (size_t)nranks;
    const CpWorkspace w = cp_workspace(d);
    if ((!x && z.x) || (!dt && z.dt) || (!B && z.bc) || (!C && z.bc) || (!y && z.x) ||
        (!records && recs_bytes))
        return SSD_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(y, 16) ||
        !aligned(records, 16) || !aligned(workspace, 16) ||
        (initial_states && !aligned(initial_states, 16)) ||
        (final_states && !aligned(final_states, 16)) || !aligned(dt, 4) || (D && !aligned(D, 4)))
        return SSD_ERR_INVALID_ARG;
    if (workspace_bytes < w.total || (w.total > 0 && !workspace)) return SSD_ERR_INVALID_ARG;
    const Range ins[] = {{x, z.x}, {dt, z.dt}, {B, z.bc}, {C, z.bc}, {D, D ? z.hv : 0},
                         {initial_states, initial_states ? z.st : 0}, {records, recs_bytes}};
    const Range outs[] = {{y, z.x}, {final_states, final_states ? z.st : 0}, {workspace, w.total}};
    for (const Range& o : outs)
        for (const Range& i : ins)
            if (overlaps(o, i)) return SSD_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i)
        for (int j = i + 1; j < 3; ++j)
            if (overlaps(outs[i], outs[j])) return SSD_ERR_INVALID_ARG;
    if (d.b * d.H * d.P * d.N > kMaxFlatStateElems) return SSD_ERR_UNSUPPORTED;
    if (d.b == 0) return SSD_OK;
    cudaStream_t s = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    const float* h_in = initial_states;
    if (rank > 0) {
        float* hin = (float*)(ws + w.off_hin);
        if ((st = cuda_status("rank fold", ssd::launch_cp_fold(d, records, (int64_t)rec_floats, rank,
                                                               hin, s))) != SSD_OK)
            return st;
        h_in = hin;
    }
    if (d.T == 0)
        return cuda_status("final states", ssd::launch_copy_or_zero_states(d, h_in, final_states, s));
    if (w.single_pass) {
        // the states entering segments 1.. from h_in, over the segment states begin left,
        // then every segment of the slice at once
        float* segbuf = (float*)(ws + w.off_seg);
        const float* decay = (const float*)(ws + w.off_decay);
        const int nslot = w.nseg + 1;
        if (w.nseg > 1 &&
            (st = cuda_status("segment scan", ssd::launch_segment_scan(d, h_in, segbuf, decay, w.nseg, nslot,
                                                                       w.nseg - 1, nullptr, s))) != SSD_OK)
            return st;
        CUtensorMap maps[4];
        if (!ssd::make_tc_maps(d, x, B, C, y, maps)) {
            ssd::set_error_detail("tensor map encoding failed");
            return SSD_ERR_CUDA;
        }
        int* sync = (int*)(ws + w.off_fwd);
        if ((st = cuda_status("sync area", cudaMemsetAsync(sync, 0, sizeof(int) * ssd::fused_sync_ints(d, w.nseg),
                                                           s))) != SSD_OK)
            return st;
        ssd::FusedLaunch a = {};
        a.d = d;
        a.maps = maps;
        a.dt = dt;
        a.A = (const float*)(ws + w.off_A);
        a.D = D;
        a.init = h_in;
        a.finalbuf = final_states;
        a.segbuf = w.nseg > 1 ? segbuf : nullptr;
        a.sync_ints = sync;
        a.kheads = ssd::fused_kheads(d.H, d.G, ssd::fused_state_capacity(d.N));
        a.seg_tiles = w.seg_tiles;
        a.nseg = w.nseg;
        a.nslot = nslot;
        a.chained = 0;
        a.y = y;
        return cuda_status("fused forward", ssd::launch_fused(a, s));
    }
    const float* cs = (const float*)(ws + w.off_cs);
    const float* S = (const float*)(ws + w.off_S);
    float* entry = (float*)(ws + w.off_entry);
    if ((st = cuda_status("state passing", ssd::launch_state_passing(d, S, cs, h_in, entry,
                                                                      final_states, s))) != SSD_OK)
        return st;
    return cuda_status("chunk scan",
                       steps_use_tc(d) ? ssd::launch_chunk_scan_tc(d, x, dt, B, C, D, cs, entry, y, s)
                                       : ssd::launch_chunk_scan_simt(d, x, dt, B, C, D, cs, entry, y, s));
}

ssd_status_t ssd_gated_rmsnorm(const ssd_shape_t* shape, const void* y, const void* z,
                               const float* weight, int64_t group_size, float eps, void* out,
                               void* stream) {
    if (!shape) return SSD_ERR_INVALID_ARG;
    ssd_shape_t s = *shape;
    s.chunk_size = 64;   // not used
    ssd_status_t st = check_shape(&s);
    if (st != SSD_OK) return st;
    const ssd::Dims d = ssd::make_dims(s);
    const int64_t C = d.H * d.P;
    if (group_size < 1 || C % group_size != 0) return SSD_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || eps > 3.0e38f) return SSD_ERR_INVALID_ARG;   // rejects NaN and inf
    const Sizes z0 = sizes_of(d);
    if ((!y && z0.x) || (!z && z0.x) || (!out && z0.x) || !weight) return SSD_ERR_INVALID_ARG;
    if (!aligned(y, 16) || !aligned(z, 16) || !aligned(out, 16) || !aligned(weight, 4))
        return SSD_ERR_INVALID_ARG;
    const Range o{out, z0.x};
    if (overlaps(o, {y, z0.x}) || overlaps(o, {z, z0.x}) || overlaps(o, {weight, (size_t)C * 4}))
        return SSD_ERR_INVALID_ARG;
    // one CTA per group at worst: keep the grid inside its x limit
    if (d.b * d.T * (C / group_size) > 2147483647LL) return SSD_ERR_UNSUPPORTED;
    return cuda_status("gated rmsnorm", ssd::launch_gated_rmsnorm(d, y, z, weight, group_size, eps, out,
                                                                  (cudaStream_t)stream));
}

ssd_status_t ssd_chunk_cumsum(const ssd_shape_t* shape, const float* dt, const float* A,
                              float* cs, void* stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (!dt || !A || !cs) return SSD_ERR_INVALID_ARG;
    const ssd::Dims d = ssd::make_dims(*shape);
    const Sizes z = sizes_of(d);
    if (overlaps({cs, z.cs}, {dt, z.dt}) || overlaps({cs, z.cs}, {A, z.hv}))
        return SSD_ERR_INVALID_ARG;
    return cuda_status("chunk cumsum", ssd::launch_chunk_cumsum(d, dt, A, cs, (cudaStream_t)stream));
}

ssd_status_t ssd_chunk_state(const ssd_shape_t* shape, const void* x, const float* dt,
                             const void* B, const float* cs, float* states, void* stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (!x || !dt || !B || !cs || !states) return SSD_ERR_INVALID_ARG;
    const ssd::Dims d = ssd::make_dims(*shape);
    const Sizes z = sizes_of(d);
    const Range o{states, z.chunk_states};
    if (overlaps(o, {x, z.x}) || overlaps(o, {dt, z.dt}) || overlaps(o, {B, z.bc}) ||
        overlaps(o, {cs, z.cs}))
        return SSD_ERR_INVALID_ARG;
    if (steps_use_tc(d))
        return cuda_status("chunk state", ssd::launch_chunk_state_tc(d, x, dt, B, cs, states,
                                                                       (cudaStream_t)stream));
    return cuda_status("chunk state", ssd::launch_chunk_state_simt(d, x, dt, B, cs, states,
                                                                     (cudaStream_t)stream));
}

ssd_status_t ssd_state_passing(const ssd_shape_t* shape, const float* states, const float* cs,
                               const float* initial_states, float* entry_states,
                               float* final_states, void* stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (!states || !cs || !entry_states) return SSD_ERR_INVALID_ARG;
    const ssd::Dims d = ssd::make_dims(*shape);
    const Sizes z = sizes_of(d);
    const Range ins[] = {{states, z.chunk_states}, {cs, z.cs},
                         {initial_states, initial_states ? z.st : 0}};
    const Range outs[] = {{entry_states, z.chunk_states}, {final_states, final_states ? z.st : 0}};
    for (const Range& o : outs)
        for (const Range& i : ins)
            if (overlaps(o, i)) return SSD_ERR_INVALID_ARG;
    if (overlaps(outs[0], outs[1])) return SSD_ERR_INVALID_ARG;
    if (d.T == 0)
        return cuda_status("final states", ssd::launch_copy_or_zero_states(d, initial_states,
                                                                           final_states,
                                                                           (cudaStream_t)stream));
    return cuda_status("state passing",
                       ssd::launch_state_passing(d, states, cs, initial_states, entry_states,
                                                 final_states, (cudaStream_t)stream));
}

ssd_status_t ssd_chunk_scan(const ssd_shape_t* shape, const void* x, const float* dt,
                            const void* B, const void* C, const float* D, const float* cs,
                            const float* entry_states, void* y, void* stream) {
    ssd_status_t st = check_shape(shape);
    if (st != SSD_OK) return st;
    if (!x || !dt || !B || !C || !cs || !entry_states || !y) return SSD_ERR_INVALID_ARG;
    const ssd::Dims d = ssd::make_dims(*shape);
    const Sizes z = sizes_of(d);
    const Range o{y, z.x};
    const Range ins[] = {{x, z.x}, {dt, z.dt}, {B, z.bc}, {C, z.bc}, {D, D ? z.hv : 0},
                         {cs, z.cs}, {entry_states, z.chunk_states}};
    for (const Range& i : ins)
        if (overlaps(o, i)) return SSD_ERR_INVALID_ARG;
    if (steps_use_tc(d))
        return cuda_status("chunk scan", ssd::launch_chunk_scan_tc(d, x, dt, B, C, D, cs,
                                                                     entry_states, y,
                                                                     (cudaStream_t)stream));
    return cuda_status("chunk scan", ssd::launch_chunk_scan_simt(d, x, dt, B, C, D, cs,
                                                                   entry_states, y,
                                                                   (cudaStream_t)stream));
}

}  // extern "C"
