// selective_scan_fwd_host: the selective scan of inputs held in host memory, with the results
// copied back to host memory, as one C call.
//
// The work is cut into pieces (groups of batch rows, or stretches of one row's sequence carried
// through the stored final state) and pipelined over three streams of the library: the
// host->device copies of piece i, the scan of piece i-1 and the device->host copy of piece i-2
// run at the same time, so both directions of the host link and the GPU are busy at once.  Each
// copy is one cudaMemcpyAsync of a contiguous block; each piece's scan is one
// selective_scan_fwd call.  The device staging buffers (two slots of one piece each) and the
// scan's workspace are carved from the caller's workspace.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "ss_internal.h"

namespace {

constexpr int kMaxDevices = 64;

// The library's streams and events for host-buffer calls on one device (created on the first
// call on that device, kept until exit).
struct HostPipe {
    cudaStream_t s_in, s_comp, s_out;
    cudaEvent_t start, fin_in, fin_comp, fin_out;
    cudaEvent_t in_done[SS_HOST_MAX_PIECES], comp_done[SS_HOST_MAX_PIECES],
        out_done[SS_HOST_MAX_PIECES];
};

std::mutex g_pipe_mutex;
HostPipe* g_pipe[kMaxDevices] = {};
std::mutex g_call_mutex[kMaxDevices];

cudaError_t host_pipe(int dev, HostPipe** out)
{
    std::lock_guard<std::mutex> lock(g_pipe_mutex);
    if (!g_pipe[dev]) {
        HostPipe* hp = new HostPipe();
        cudaError_t e = cudaSuccess;
        const unsigned ef = cudaEventDisableTiming;
        for (cudaStream_t* s : {&hp->s_in, &hp->s_comp, &hp->s_out})
            if (e == cudaSuccess)
                e = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking);
        for (cudaEvent_t* ev : {&hp->start, &hp->fin_in, &hp->fin_comp, &hp->fin_out})
            if (e == cudaSuccess)
                e = cudaEventCreateWithFlags(ev, ef);
        for (int i = 0; i < SS_HOST_MAX_PIECES && e == cudaSuccess; ++i) {
            e = cudaEventCreateWithFlags(&hp->in_done[i], ef);
            if (e == cudaSuccess)
                e = cudaEventCreateWithFlags(&hp->comp_done[i], ef);
            if (e == cudaSuccess)
                e = cudaEventCreateWithFlags(&hp->out_done[i], ef);
        }
        if (e != cudaSuccess) {
            delete hp;  // (streams or events already created are not reclaimed on this path)
            return e;
        }
        g_pipe[dev] = hp;
    }
    *out = g_pipe[dev];
    return cudaSuccess;
}

struct Piece {
    int64_t r0, r1;  // batch rows r0..r1-1
    int64_t a, b;    // steps a..b-1
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct HostPlan {
    int64_t batch, L, D, N;
    int K, esz, dsz;
    bool u_per_dir, carry, has_z, has_init;
    int np;
    Piece pc[SS_HOST_MAX_PIECES];
    int64_t rows_max, steps_max;
    // one staging slot (byte offsets); the scan workspace follows the two slots
    size_t off_u, off_d, off_B, off_C, off_z, off_out, off_last, off_init, slot_bytes;
    size_t scan_ws, bytes;
};

ss_status make_host_plan(const ss_shape* s, const ss_direction_map* dmap,
                         const ss_launch_opts* opts, int32_t pieces, HostPlan* hp)
{
    size_t ws = 0;
    ss_status st = selective_scan_workspace_size(s, dmap, opts, &ws);  // validates everything
    if (st != SS_OK)
        return st;
    if (pieces < 1 || pieces > SS_HOST_MAX_PIECES)
        return SS_ERR_UNSUPPORTED;
    const int flags = opts ? opts->flags : 0;
    hp->batch = s->batch;
    hp->L = s->seqlen;
    hp->D = s->dim;
    hp->N = s->dstate;
    hp->K = dmap ? dmap->num_dirs : 1;
    hp->esz = s->io_dtype == SS_BF16 ? 2 : 4;
    hp->dsz = (flags & SS_FLAG_DELTA_INT8) ? 1 : hp->esz;
    hp->u_per_dir = (flags & SS_FLAG_U_PER_DIRECTION) != 0;
    hp->has_init = opts && opts->initial_state;
    const bool conv = opts && opts->conv_weight;
    const bool fwd_only = hp->K == 1 && (!dmap || dmap->dir[0] == SS_DIR_FWD);
    // sequence pieces need a state carried from piece to piece: one forward direction, and no
    // convolution (whose window would reach into the previous piece)
    hp->carry = fwd_only && !conv && !hp->u_per_dir && hp->L > 0 &&
                (hp->batch == 1 || pieces > hp->batch);
    hp->np = 0;
    if (hp->batch > 0 && hp->L > 0 && hp->D > 0) {
        if (hp->carry) {
            const int64_t parts = (pieces + hp->batch - 1) / hp->batch;
            int64_t step = (hp->L + parts - 1) / parts;
            step = ((step + ss::kTile - 1) / ss::kTile) * ss::kTile;  // whole tiles
            for (int64_t r = 0; r < hp->batch; ++r)
                for (int64_t a = 0; a < hp->L; a += step) {
                    if (hp->np >= SS_HOST_MAX_PIECES)
                        return SS_ERR_UNSUPPORTED;
                    hp->pc[hp->np++] = Piece{r, r + 1, a, (a + step < hp->L) ? a + step : hp->L};
                }
        } else {
            const int64_t nb = pieces < hp->batch ? pieces : hp->batch;
            const int64_t rstep = (hp->batch + nb - 1) / nb;
            for (int64_t r = 0; r < hp->batch; r += rstep)
                hp->pc[hp->np++] = Piece{r, (r + rstep < hp->batch) ? r + rstep : hp->batch, 0, hp->L};
        }
    }
    hp->rows_max = hp->steps_max = 0;
    for (int i = 0; i < hp->np; ++i) {
        const int64_t rows = hp->pc[i].r1 - hp->pc[i].r0, steps = hp->pc[i].b - hp->pc[i].a;
        hp->rows_max = rows > hp->rows_max ? rows : hp->rows_max;
        hp->steps_max = steps > hp->steps_max ? steps : hp->steps_max;
    }
    const size_t rl = static_cast<size_t>(hp->rows_max) * hp->steps_max;
    const size_t Ku = hp->u_per_dir ? hp->K : 1;
    size_t off = 0;
    hp->off_u = off;
    off = align256(off + Ku * rl * hp->D * hp->esz);
    hp->off_d = off;
    off = align256(off + hp->K * rl * hp->D * hp->dsz);
    hp->off_B = off;
    off = align256(off + hp->K * rl * hp->N * hp->esz);
    hp->off_C = off;
    off = align256(off + hp->K * rl * hp->N * hp->esz);
    hp->off_z = off;
    off = align256(off + rl * hp->D * hp->esz);  // (unused without z)
    hp->off_out = off;
    off = align256(off + rl * hp->D * hp->esz);
    hp->off_last = off;
    off = align256(off + static_cast<size_t>(hp->K) * hp->rows_max * hp->D * hp->N * 4);
    hp->off_init = off;
    off = align256(off + (hp->has_init ? static_cast<size_t>(hp->K) * hp->rows_max * hp->D * hp->N * 4 : 0));
    hp->slot_bytes = off;
    // the scan workspace of the largest piece shape (pieces scan one after another)
    hp->scan_ws = 0;
    for (int i = 0; i < hp->np; ++i) {
        ss_shape ps = *s;
        ps.batch = hp->pc[i].r1 - hp->pc[i].r0;
        ps.seqlen = hp->pc[i].b - hp->pc[i].a;
        size_t w = 0;
        st = selective_scan_workspace_size(&ps, dmap, opts, &w);
        if (st != SS_OK)
            return st;
        hp->scan_ws = w > hp->scan_ws ? w : hp->scan_ws;
    }
    hp->bytes = hp->np > 0 ? 2 * hp->slot_bytes + align256(hp->scan_ws) : 0;
    return SS_OK;
}

}  // namespace

extern "C" {

ss_status selective_scan_host_workspace_size(const ss_shape* shape, const ss_direction_map* dmap,
                                             const ss_launch_opts* opts, int32_t pieces,
                                             size_t* bytes)
{
    if (!bytes)
        return SS_ERR_NULL;
    HostPlan hp;
    const ss_status st = make_host_plan(shape, dmap, opts, pieces, &hp);
    if (st != SS_OK)
        return st;
    *bytes = hp.bytes;
    return SS_OK;
}

ss_status selective_scan_fwd_host(const ss_shape* shape, const void* u, const void* delta,
                                  const float* A, const void* B, const void* C, const float* Dskip,
                                  const void* z, const float* delta_bias, int32_t softplus,
                                  const ss_direction_map* dmap, void* out, float* last_state,
                                  void* workspace, size_t workspace_bytes, int32_t pieces,
                                  void* stream, const ss_launch_opts* opts)
{
    HostPlan hp;
    ss_status st = make_host_plan(shape, dmap, opts, pieces, &hp);
    if (st != SS_OK)
        return st;
    const bool has_data = hp.batch * hp.L * hp.D > 0;
    if (has_data && (!u || !delta || !B || !C || !out))
        return SS_ERR_NULL;
    if (hp.K * hp.batch * hp.D > 0 && !A)
        return SS_ERR_NULL;
    if (hp.bytes > 0 && (!workspace || workspace_bytes < hp.bytes))
        return SS_ERR_WORKSPACE;
    if (workspace && reinterpret_cast<uintptr_t>(workspace) % 256 != 0)
        return SS_ERR_ALIGN;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return SS_ERR_CUDA;
    cudaStream_t caller = static_cast<cudaStream_t>(stream);
    int sdev = dev;
    if (cudaStreamGetDevice(caller, &sdev) != cudaSuccess)
        return SS_ERR_CUDA;
    if (sdev != dev)
        return SS_ERR_DEVICE;
    HostPipe* pp = nullptr;
    if (host_pipe(dev, &pp) != cudaSuccess)
        return SS_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_call_mutex[dev]);

    const int K = hp.K;
    const int64_t L = hp.L, D = hp.D, N = hp.N, batch = hp.batch;
    const size_t esz = hp.esz, dsz = hp.dsz;
    const bool want_last = last_state != nullptr;
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    const unsigned char* hu = static_cast<const unsigned char*>(u);
    const unsigned char* hd = static_cast<const unsigned char*>(delta);
    const unsigned char* hB = static_cast<const unsigned char*>(B);
    const unsigned char* hC = static_cast<const unsigned char*>(C);
    const unsigned char* hz = static_cast<const unsigned char*>(z);
    unsigned char* ho = static_cast<unsigned char*>(out);
    unsigned char* hl = reinterpret_cast<unsigned char*>(last_state);
    const float* init = opts ? opts->initial_state : nullptr;

#define SS_TRY(x)                      \
    do {                               \
        if ((x) != cudaSuccess)        \
            return SS_ERR_CUDA;        \
    } while (0)

    // everything follows the work already on the caller's stream
    SS_TRY(cudaEventRecord(pp->start, caller));
    SS_TRY(cudaStreamWaitEvent(pp->s_in, pp->start, 0));
    SS_TRY(cudaStreamWaitEvent(pp->s_comp, pp->start, 0));
    SS_TRY(cudaStreamWaitEvent(pp->s_out, pp->start, 0));

    if (!has_data) {
        // no step is taken: the final state is the initial state (zero when none is given)
        if (want_last && K * batch * D > 0) {
            const size_t n = static_cast<size_t>(K) * batch * D * N * sizeof(float);
            if (init)
                SS_TRY(cudaMemcpyAsync(last_state, init, n, cudaMemcpyDeviceToHost, pp->s_out));
            else
                std::memset(last_state, 0, n);  // (nothing of the call reads it on the device)
        }
    }

    auto H2D = [&](void* dst, const void* src, size_t n) {
        return n ? cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, pp->s_in) : cudaSuccess;
    };
    auto D2H = [&](void* dst, const void* src, size_t n) {
        return n ? cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToHost, pp->s_out) : cudaSuccess;
    };
    // Copy rows r0..r1-1, steps a..b-1 of a host tensor [blocks, batch, L, W] (element size es)
    // into the device tensor [blocks, rows, steps, W]: one copy per block when the steps are
    // whole rows, else one per (block, row).
    auto in_block = [&](unsigned char* dst, const unsigned char* src, int blocks, const Piece& pc,
                        int64_t W, size_t es) {
        const int64_t rows = pc.r1 - pc.r0, steps = pc.b - pc.a;
        for (int kk = 0; kk < blocks; ++kk) {
            const unsigned char* sk = src + static_cast<size_t>(kk) * batch * L * W * es;
            unsigned char* dk = dst + static_cast<size_t>(kk) * rows * steps * W * es;
            if (steps == L) {
                if (H2D(dk, sk + static_cast<size_t>(pc.r0) * L * W * es,
                        static_cast<size_t>(rows) * L * W * es) != cudaSuccess)
                    return cudaErrorUnknown;
            } else {
                for (int64_t r = 0; r < rows; ++r)
                    if (H2D(dk + static_cast<size_t>(r) * steps * W * es,
                            sk + (static_cast<size_t>(pc.r0 + r) * L + pc.a) * W * es,
                            static_cast<size_t>(steps) * W * es) != cudaSuccess)
                        return cudaErrorUnknown;
            }
        }
        return cudaSuccess;
    };

    for (int i = 0; i < hp.np; ++i) {
        const Piece& pc = hp.pc[i];
        const int slot = i & 1;
        unsigned char* sb = ws + slot * hp.slot_bytes;
        const int64_t rows = pc.r1 - pc.r0, steps = pc.b - pc.a;
        // ---- copies in (after the scan of piece i-2, which read this slot)
        if (i >= 2)
            SS_TRY(cudaStreamWaitEvent(pp->s_in, pp->comp_done[i - 2], 0));
        SS_TRY(in_block(sb + hp.off_u, hu, hp.u_per_dir ? K : 1, pc, D, esz));
        SS_TRY(in_block(sb + hp.off_d, hd, K, pc, D, dsz));
        SS_TRY(in_block(sb + hp.off_B, hB, K, pc, N, esz));
        SS_TRY(in_block(sb + hp.off_C, hC, K, pc, N, esz));
        if (z)
            SS_TRY(in_block(sb + hp.off_z, hz, 1, pc, D, esz));
        SS_TRY(cudaEventRecord(pp->in_done[i], pp->s_in));
        // ---- scan (after its inputs, and after the copy out of piece i-2's output slot)
        SS_TRY(cudaStreamWaitEvent(pp->s_comp, pp->in_done[i], 0));
        if (i >= 2)
            SS_TRY(cudaStreamWaitEvent(pp->s_comp, pp->out_done[i - 2], 0));
        ss_launch_opts po;
        std::memset(&po, 0, sizeof(po));
        if (opts)
            po = *opts;
        po.scan_begin_event = po.scan_end_event = nullptr;
        float* last_dev = reinterpret_cast<float*>(sb + hp.off_last);
        if (hp.carry && pc.a > 0) {
            // continue from the previous piece of this row (the other slot)
            po.initial_state = reinterpret_cast<float*>(ws + (slot ^ 1) * hp.slot_bytes + hp.off_last);
        } else if (init) {
            float* init_dev = reinterpret_cast<float*>(sb + hp.off_init);
            for (int kk = 0; kk < K; ++kk)
                SS_TRY(cudaMemcpyAsync(init_dev + static_cast<size_t>(kk) * rows * D * N,
                                       init + (static_cast<size_t>(kk) * batch + pc.r0) * D * N,
                                       static_cast<size_t>(rows) * D * N * sizeof(float),
                                       cudaMemcpyDeviceToDevice, pp->s_comp));
            po.initial_state = init_dev;
        } else {
            po.initial_state = nullptr;
        }
        const bool last_piece_of_row = pc.b == L;
        const bool need_last = hp.carry || (want_last && last_piece_of_row);
        ss_shape ps = *shape;
        ps.batch = rows;
        ps.seqlen = steps;
        st = selective_scan_fwd(&ps, sb + hp.off_u, sb + hp.off_d, A, sb + hp.off_B, sb + hp.off_C,
                                Dskip, z ? sb + hp.off_z : nullptr, delta_bias, softplus, dmap,
                                sb + hp.off_out, need_last ? last_dev : nullptr,
                                hp.scan_ws ? ws + 2 * hp.slot_bytes : nullptr, hp.scan_ws,
                                pp->s_comp, &po);
        if (st != SS_OK)
            return st;
        SS_TRY(cudaEventRecord(pp->comp_done[i], pp->s_comp));
        // ---- copies out
        SS_TRY(cudaStreamWaitEvent(pp->s_out, pp->comp_done[i], 0));
        const unsigned char* od = sb + hp.off_out;
        if (steps == L) {
            SS_TRY(D2H(ho + static_cast<size_t>(pc.r0) * L * D * esz, od,
                       static_cast<size_t>(rows) * L * D * esz));
        } else {
            for (int64_t r = 0; r < rows; ++r)
                SS_TRY(D2H(ho + (static_cast<size_t>(pc.r0 + r) * L + pc.a) * D * esz,
                           od + static_cast<size_t>(r) * steps * D * esz,
                           static_cast<size_t>(steps) * D * esz));
        }
        if (want_last && last_piece_of_row)
            for (int kk = 0; kk < K; ++kk)
                SS_TRY(D2H(hl + (static_cast<size_t>(kk) * batch + pc.r0) * D * N * sizeof(float),
                           last_dev + static_cast<size_t>(kk) * rows * D * N,
                           static_cast<size_t>(rows) * D * N * sizeof(float)));
        SS_TRY(cudaEventRecord(pp->out_done[i], pp->s_out));
    }
    // the caller's stream continues after every copy and scan of the call
    SS_TRY(cudaEventRecord(pp->fin_in, pp->s_in));
    SS_TRY(cudaEventRecord(pp->fin_comp, pp->s_comp));
    SS_TRY(cudaEventRecord(pp->fin_out, pp->s_out));
    SS_TRY(cudaStreamWaitEvent(caller, pp->fin_in, 0));
    SS_TRY(cudaStreamWaitEvent(caller, pp->fin_comp, 0));
    SS_TRY(cudaStreamWaitEvent(caller, pp->fin_out, 0));
#undef SS_TRY
    return SS_OK;
}

}  // extern "C"
