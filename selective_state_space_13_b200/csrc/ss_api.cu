// Host entry points of the selective scan library (the C ABI of include/selective_scan.h):
// argument validation, workspace sizing, segment choice and the launch sequence.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "ss_internal.h"

namespace {

constexpr int64_t kMaxSeqlen = (int64_t{1} << 31) - 1;
// Automatic segment choice (measured on B200): when the (direction, batch row, channel tile)
// units give fewer than about 1.5 CTAs per SM, split each sequence into S segments so that the
// scan launch's units * S CTAs fill one wave of the kWaveCtas resident slots (6 CTAs on each
// of the 148 SMs) as closely as possible without starting a second, mostly idle wave; when the
// segments would still exceed kLongSegSteps steps, S is multiplied up to whole waves again.
// Segments never go below kMinSegSteps steps.  (With more units the segment-aggregate launch
// costs more than the parallelism it adds.)  Measured: m130 -> 4, long -> 22, cromb -> 18;
// long runs 4.17 ms at 22 segments against 4.54 at 14.  The slot count is that of B200, so
// that the plan (and the workspace size) never depends on the device present.
constexpr int64_t kSplitBelowCtas = 222;
constexpr int64_t kWaveCtas = 6 * 148;
constexpr int64_t kLongSegSteps = 8192;
constexpr int64_t kMinSegSteps = 16 * ss::kTile;
constexpr int kMaxSegments = 1024;

struct Plan {
    int64_t batch, L, D, N;
    int io;
    int K;
    int32_t dirs[SS_MAX_DIRS];
    int32_t H, W;
    int S;
    int64_t seg_len;
    int flags;
    cudaEvent_t ev_begin, ev_end;
    const float* init_state;
    const float* conv_w;
    const float* conv_b;
    int conv_width;
    const float* delta_scale;
    // workspace layout (byte offsets, 0 size = unused)
    size_t off_carry_h, off_carry_s, off_ypart, bytes;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

ss_status make_plan(const ss_shape* s, const ss_direction_map* dmap, const ss_launch_opts* opts,
                    Plan* pl)
{
    if (!s)
        return SS_ERR_NULL;
    if (s->reserved != 0)
        return SS_ERR_SHAPE;
    if (s->io_dtype != SS_F32 && s->io_dtype != SS_BF16)
        return SS_ERR_DTYPE;
    if (s->batch < 0 || s->seqlen < 0 || s->dim < 0 || s->seqlen > kMaxSeqlen)
        return SS_ERR_SHAPE;
    if (s->dstate < 1)
        return SS_ERR_SHAPE;
    if (s->dstate > SS_MAX_DSTATE)
        return SS_ERR_UNSUPPORTED;
    if (s->batch > (int64_t{1} << 24) || s->dim > (int64_t{1} << 24))
        return SS_ERR_SHAPE;
    // tile coordinates are 32-bit: every direction's rows must be addressable; a position's
    // element offset inside one sequence (L * D) must fit in 32 bits as well
    if (s->batch * s->seqlen * SS_MAX_DIRS > kMaxSeqlen || s->seqlen * s->dim > kMaxSeqlen)
        return SS_ERR_SHAPE;
    const int esz = s->io_dtype == SS_BF16 ? 2 : 4;
    if ((s->dim * esz) % 16 != 0)
        return SS_ERR_ALIGN;

    pl->batch = s->batch;
    pl->L = s->seqlen;
    pl->D = s->dim;
    pl->N = s->dstate;
    pl->io = s->io_dtype;
    pl->H = 0;
    pl->W = 0;
    for (int k = 0; k < SS_MAX_DIRS; ++k)
        pl->dirs[k] = SS_DIR_FWD;
    if (!dmap) {
        pl->K = 1;
    } else {
        if (dmap->num_dirs < 1 || dmap->num_dirs > SS_MAX_DIRS)
            return SS_ERR_DIRMAP;
        pl->K = dmap->num_dirs;
        bool col = false;
        for (int k = 0; k < pl->K; ++k) {
            const int32_t d = dmap->dir[k];
            if (d < SS_DIR_FWD || d > SS_DIR_COL_REV)
                return SS_ERR_DIRMAP;
            pl->dirs[k] = d;
            col = col || d == SS_DIR_COL || d == SS_DIR_COL_REV;
        }
        if (col) {
            if (dmap->H <= 0 || dmap->W <= 0 ||
                static_cast<int64_t>(dmap->H) * static_cast<int64_t>(dmap->W) != s->seqlen)
                return SS_ERR_DIRMAP;
        }
        pl->H = dmap->H;
        pl->W = dmap->W;
    }

    int seg = 0;
    pl->flags = 0;
    pl->ev_begin = pl->ev_end = nullptr;
    pl->init_state = nullptr;
    pl->conv_w = pl->conv_b = nullptr;
    pl->conv_width = 0;
    pl->delta_scale = nullptr;
    if (opts) {
        if (opts->reserved != 0)
            return SS_ERR_UNSUPPORTED;
        if (opts->conv_weight) {
            if (opts->conv_width < 1 || opts->conv_width > SS_MAX_CONV_WIDTH)
                return SS_ERR_UNSUPPORTED;
        } else if (opts->conv_bias || opts->conv_width != 0) {
            return SS_ERR_UNSUPPORTED;
        }
        pl->conv_w = opts->conv_weight;
        pl->conv_b = opts->conv_bias;
        pl->conv_width = opts->conv_weight ? opts->conv_width : 0;
        if (opts->segments < 0 || opts->segments > kMaxSegments)
            return SS_ERR_UNSUPPORTED;
        if (opts->flags & ~(SS_FLAG_GENERIC_A | SS_FLAG_ZOH_EXACT | SS_FLAG_TEST_WAIT_TIMEOUT |
                            SS_FLAG_U_PER_DIRECTION | SS_FLAG_DELTA_INT8 |
                            SS_FLAG_PARAMS_PER_DIRECTION))
            return SS_ERR_UNSUPPORTED;
        if (opts->flags & SS_FLAG_DELTA_INT8) {
            if (s->io_dtype != SS_BF16)
                return SS_ERR_UNSUPPORTED;
            if (!opts->delta_scale)
                return SS_ERR_NULL;
            if (s->dim % 16 != 0)
                return SS_ERR_ALIGN;
            pl->delta_scale = opts->delta_scale;
        } else if (opts->delta_scale) {
            return SS_ERR_UNSUPPORTED;
        }
        pl->init_state = opts->initial_state;
        seg = opts->segments;
        pl->flags = opts->flags;
        pl->ev_begin = static_cast<cudaEvent_t>(opts->scan_begin_event);
        pl->ev_end = static_cast<cudaEvent_t>(opts->scan_end_event);
    }
    const int64_t L = pl->L;
    if (L == 0) {
        seg = 1;
    } else if (seg == 0) {
        const int64_t ctas = ((pl->D + ss::channels_per_cta() - 1) / ss::channels_per_cta()) *
                             pl->batch * pl->K;
        seg = 1;
        if (ctas > 0 && ctas < kSplitBelowCtas) {
            int64_t want = kWaveCtas / ctas;  // >= 4: ctas < kSplitBelowCtas
            const int64_t waves = (L + want * kLongSegSteps - 1) / (want * kLongSegSteps);
            if (waves > 1)
                want *= waves;
            const int64_t cap = L / kMinSegSteps;
            if (want > cap)
                want = cap;
            if (want > kMaxSegments)
                want = kMaxSegments;
            seg = want > 1 ? static_cast<int>(want) : 1;
        }
    }
    if (seg > L && L > 0)
        seg = static_cast<int>(L);
    // equal segments, a multiple of the tile long (the last one takes the remainder)
    int64_t seg_len = (L + seg - 1) / seg;
    seg_len = ((seg_len + ss::kTile - 1) / ss::kTile) * ss::kTile;
    if (seg_len == 0)
        seg_len = ss::kTile;
    pl->S = static_cast<int>((L + seg_len - 1) / seg_len);
    if (pl->S < 1)
        pl->S = 1;
    pl->seg_len = seg_len;

    size_t off = 0;
    pl->off_carry_h = pl->off_carry_s = pl->off_ypart = 0;
    if (pl->S > 1) {
        // fp32 inputs carry their segment states in fp64 (the precise kernel's state type)
        const size_t cells = static_cast<size_t>(pl->K) * pl->batch * pl->S * pl->D;
        const size_t cb = pl->io == SS_F32 ? sizeof(double) : sizeof(float);
        pl->off_carry_h = off;
        off = align256(off + cells * pl->N * cb);
        pl->off_carry_s = off;
        off = align256(off + cells * cb);
    }
    if (pl->K > 1) {
        pl->off_ypart = off;
        off = align256(off + static_cast<size_t>(pl->K) * pl->batch * pl->L * pl->D * sizeof(float));
    }
    pl->bytes = off;
    return SS_OK;
}

}  // namespace

extern "C" {

ss_status selective_scan_workspace_size(const ss_shape* shape, const ss_direction_map* dmap,
                                        const ss_launch_opts* opts, size_t* bytes)
{
    if (!bytes)
        return SS_ERR_NULL;
    Plan pl;
    const ss_status st = make_plan(shape, dmap, opts, &pl);
    if (st != SS_OK)
        return st;
    *bytes = pl.bytes;
    return SS_OK;
}

ss_status selective_scan_fwd(const ss_shape* shape, const void* u, const void* delta,
                             const float* A, const void* B, const void* C, const float* Dskip,
                             const void* z, const float* delta_bias, int32_t softplus,
                             const ss_direction_map* dmap, void* out, float* last_state,
                             void* workspace, size_t workspace_bytes, void* stream,
                             const ss_launch_opts* opts)
{
    Plan pl;
    ss_status st = make_plan(shape, dmap, opts, &pl);
    if (st != SS_OK)
        return st;
    const bool has_data = pl.batch * pl.L * pl.D > 0;
    const bool has_state = pl.K * pl.batch * pl.D > 0;
    if (has_data && (!u || !delta || !B || !C || !out))
        return SS_ERR_NULL;
    if (has_state && !A)
        return SS_ERR_NULL;
    for (const void* p : {u, delta, B, C, z, static_cast<const void*>(out),
                          static_cast<const void*>(workspace)})
        if (p && !aligned(p, 16))
            return SS_ERR_ALIGN;
    for (const void* p : {static_cast<const void*>(A), static_cast<const void*>(Dskip),
                          static_cast<const void*>(delta_bias), static_cast<const void*>(last_state),
                          static_cast<const void*>(pl.init_state),
                          static_cast<const void*>(pl.conv_w), static_cast<const void*>(pl.conv_b),
                          static_cast<const void*>(pl.delta_scale)})
        if (p && !aligned(p, 4))
            return SS_ERR_ALIGN;
    if (pl.bytes > 0 && (!workspace || workspace_bytes < pl.bytes))
        return SS_ERR_WORKSPACE;

    cudaStream_t strm = static_cast<cudaStream_t>(stream);
    // the stream must belong to the current device, whose error word the kernels report to
    auto stream_on_current_device = [&]() -> ss_status {
        int dev = 0, sdev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaStreamGetDevice(strm, &sdev) != cudaSuccess)
            return SS_ERR_CUDA;
        return sdev == dev ? SS_OK : SS_ERR_DEVICE;
    };
    if (!has_data) {
        // no step is taken: the final state is the initial state (zero when none is given)
        if (last_state && has_state && pl.L == 0) {
            if ((st = stream_on_current_device()) != SS_OK)
                return st;
            const size_t n = static_cast<size_t>(pl.K) * pl.batch * pl.D * pl.N * sizeof(float);
            const cudaError_t e =
                pl.init_state
                    ? cudaMemcpyAsync(last_state, pl.init_state, n, cudaMemcpyDeviceToDevice, strm)
                    : cudaMemsetAsync(last_state, 0, n, strm);
            if (e != cudaSuccess)
                return SS_ERR_CUDA;
        }
        return SS_OK;
    }

    if ((st = stream_on_current_device()) != SS_OK)
        return st;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    ss::ScanParams p;
    std::memset(&p, 0, sizeof(p));
    p.u = u;
    p.delta = delta;
    p.A = A;
    p.B = B;
    p.C = C;
    p.Dskip = Dskip;
    p.z = z;
    p.bias = delta_bias;
    p.out = out;
    p.ypart = pl.K > 1 ? reinterpret_cast<float*>(ws + pl.off_ypart) : nullptr;
    p.last_state = last_state;
    p.carry_h = pl.S > 1 ? reinterpret_cast<float*>(ws + pl.off_carry_h) : nullptr;
    p.carry_s = pl.S > 1 ? reinterpret_cast<float*>(ws + pl.off_carry_s) : nullptr;
    p.batch = pl.batch;
    p.L = pl.L;
    p.D = pl.D;
    p.seg_len = pl.seg_len;
    p.N = static_cast<int32_t>(pl.N);
    p.K = pl.K;
    p.S = pl.S;
    for (int k = 0; k < SS_MAX_DIRS; ++k)
        p.dirs[k] = pl.dirs[k];
    p.H = pl.H;
    p.W = pl.W;
    p.softplus = softplus ? 1 : 0;
    p.force_generic = (pl.flags & SS_FLAG_GENERIC_A) ? 1 : 0;
    p.zoh = (pl.flags & SS_FLAG_ZOH_EXACT) ? 1 : 0;
    p.test_timeout = (pl.flags & SS_FLAG_TEST_WAIT_TIMEOUT) ? 1 : 0;
    p.u_per_dir = (pl.flags & SS_FLAG_U_PER_DIRECTION) ? 1 : 0;
    p.params_per_dir = (pl.flags & SS_FLAG_PARAMS_PER_DIRECTION) ? 1 : 0;
    p.status = ss::status_word();
    if (!p.status)
        return SS_ERR_CUDA;
    p.init_state = pl.init_state;
    p.conv_w = pl.conv_w;
    p.conv_b = pl.conv_b;
    p.conv_width = pl.conv_width;
    p.delta_scale = pl.delta_scale;

    // tensor maps and kernel attributes for every launch of the call, before the first one
    if (ss::prepare_scan(p, pl.io) != cudaSuccess)
        return SS_ERR_CUDA;
    // the timing events bracket the scan pipeline: the segment-aggregate launch (if any) and
    // the scan launch, which may overlap (nothing is recorded between them)
    if (pl.ev_begin && cudaEventRecord(pl.ev_begin, strm) != cudaSuccess)
        return SS_ERR_CUDA;
    if (pl.S > 1 && ss::launch_scan(p, pl.io, 1, strm) != cudaSuccess)
        return SS_ERR_CUDA;
    if (ss::launch_scan(p, pl.io, 0, strm) != cudaSuccess)
        return SS_ERR_CUDA;
    if (pl.ev_end && cudaEventRecord(pl.ev_end, strm) != cudaSuccess)
        return SS_ERR_CUDA;
    if (pl.K > 1) {
        ss::MergeParams m;
        m.ypart = p.ypart;
        m.z = z;
        m.out = out;
        m.rows = pl.batch * pl.L;
        m.D = pl.D;
        m.K = pl.K;
        if (ss::launch_merge(m, pl.io, strm) != cudaSuccess)
            return SS_ERR_CUDA;
    }
    return SS_OK;
}

int64_t ss_direction_position(const ss_direction_map* dmap, int32_t k, int64_t L, int64_t t)
{
    if (L <= 0 || t < 0 || t >= L || L > kMaxSeqlen)
        return -1;
    if (!dmap)
        return k == 0 ? t : -1;
    if (k < 0 || k >= dmap->num_dirs || dmap->num_dirs > SS_MAX_DIRS)
        return -1;
    const int32_t d = dmap->dir[k];
    if (d < SS_DIR_FWD || d > SS_DIR_COL_REV)
        return -1;
    if ((d == SS_DIR_COL || d == SS_DIR_COL_REV) &&
        (dmap->H <= 0 || dmap->W <= 0 || static_cast<int64_t>(dmap->H) * dmap->W != L))
        return -1;
    return ss::position_host(d, L, dmap->H, dmap->W, t);
}

ss_status selective_scan_device_status(void* stream, int32_t clear)
{
    unsigned int v = 0;
    if (ss::read_status(static_cast<cudaStream_t>(stream), clear != 0, &v) != cudaSuccess)
        return SS_ERR_CUDA;
    return v ? SS_ERR_DEVICE_TIMEOUT : SS_OK;
}

const char* ss_status_str(ss_status status)
{
    switch (status) {
    case SS_OK: return "SS_OK";
    case SS_ERR_NULL: return "SS_ERR_NULL: a required pointer is NULL";
    case SS_ERR_SHAPE: return "SS_ERR_SHAPE: invalid or inconsistent sizes";
    case SS_ERR_DTYPE: return "SS_ERR_DTYPE: io_dtype must be SS_F32 or SS_BF16";
    case SS_ERR_ALIGN: return "SS_ERR_ALIGN: pointer or row pitch breaks the 16-byte rule";
    case SS_ERR_DIRMAP: return "SS_ERR_DIRMAP: invalid direction map";
    case SS_ERR_UNSUPPORTED: return "SS_ERR_UNSUPPORTED: dstate or option not supported";
    case SS_ERR_CUDA: return "SS_ERR_CUDA: the CUDA runtime reported an error";
    case SS_ERR_WORKSPACE: return "SS_ERR_WORKSPACE: workspace missing or too small";
    case SS_ERR_DEVICE_TIMEOUT: return "SS_ERR_DEVICE_TIMEOUT: a kernel gave up a bounded wait";
    case SS_ERR_SCRATCH_LIMIT:
        return "SS_ERR_SCRATCH_LIMIT: the problem needs more scratch than SS_NOALLOC_SCRATCH_BYTES";
    case SS_ERR_DEVICE:
        return "SS_ERR_DEVICE: the stream belongs to another device than the current one";
    }
    return "unknown ss_status";
}

int32_t ss_abi_version(void) { return SS_ABI_VERSION; }

}  // extern "C"
