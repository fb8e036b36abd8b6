// Selective scan (S6) forward kernels for sm_100a.
//
// One thread owns one channel d of one (batch row, direction, segment) and keeps that channel's
// N-state vector in registers for the whole segment ("Understanding Mamba from zero" sec. 5:
// per channel and per state the recurrence is the scalar affine map h_t = a_t h_{t-1} + b_t).
// A CTA of 32*WARPS threads owns a tile of adjacent channels.  Its inputs stream through a
// ring of kStages shared-memory stages of kTile steps each; warp 0 fills the ring with bulk
// asynchronous copies (TMA, cp.async.bulk) that complete on an mbarrier, one copy per row of
// u / z (rows picked through the direction's index map) and delta (scan order), plus one copy
// each for the B and C tiles, which every channel of the CTA shares.  B and C are converted to
// fp32 once per CTA per stage.  Everything of a step -- softplus, exp, the recurrence, the C
// readout, the D skip and the silu gate -- happens in registers; each input element is read
// from HBM once and each output element written once.
//
// Two algebraic rewrites keep the per-update work at three FP32 operations:
//  * exp-power chain: when A[d,n] = (n+1) * A[d,0] for every n (checked in the kernel, per
//    channel), exp(Delta*A[d,n]) = q^(n+1) with q = exp(Delta*A[d,0]): one MUFU ex2 per step and
//    one multiply per state instead of one ex2 per state.
//  * normalised state k = h / w with w = Delta*u: the update h = Abar*h + w*B becomes
//    k = (w_prev/w)*Abar*k + B and y = w * (C . k), which drops the per-state w*B product.
//    |w| is clamped below at 2^-64; this changes the B term of such a step by at most
//    2^-64*|B| in absolute value.
//  All exponentials run in base 2: x is carried as (delta+bias)*log2(e), so softplus in base 2
//  gives Delta*log2(e) directly, exp(Delta*A) = ex2(Delta*log2(e) * A), and the missing ln 2
//  of w = Delta*u is folded into the fp32 copy of B.
//
// Long sequences are split into S segments (the chunked scan of "S4 -> Mamba" sec. 2.2): a
// first launch scans segments 0..S-2 from a zero state and stores each end state and the
// segment's sum of Delta; the second launch starts segment s from the carry obtained by
// folding the carries of segments 0..s-1 with the affine combine (P2, h2) o (P1, h1) =
// (P2*P1, P2*h1 + h2), P = exp(A * sum Delta).
//
// Every wait on an mbarrier is bounded in time.  A wait that gives up sets the library's device
// error word (read by selective_scan_device_status), waits a bounded time for the copies this
// CTA still has in flight, and the whole CTA returns.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ss_internal.h"

namespace ss {

__device__ unsigned int g_ss_status = 0;

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kTinyW = 5.421010862427522e-20f;  // 2^-64
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s
constexpr unsigned int kStatusTimeout = 1u;

// ---------------------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile(
        "{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase with this parity to complete, for at most limit_ns.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  unsigned long long limit_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 31u) == 0u && global_ns() - t0 > limit_ns)
            return false;
    }
}

// Bulk asynchronous copy global -> shared; completes `bytes` of transaction on `bar`.
// dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float lg2(float x)
{
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------------------------- element types

template <typename T> struct Io;
template <> struct Io<float> {
    static __device__ __forceinline__ float ld(const float* p) { return *p; }
    static __device__ __forceinline__ float st(float v) { return v; }
};
template <> struct Io<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16* p)
    {
        const unsigned short bits = *reinterpret_cast<const unsigned short*>(p);
        return __uint_as_float(static_cast<uint32_t>(bits) << 16);
    }
    static __device__ __forceinline__ __nv_bfloat16 st(float v) { return __float2bfloat16_rn(v); }
};

// ---------------------------------------------------------------------------- index map

// Spatial position visited at step t of a scan in direction dir over L = H*W positions laid
// out row by row.  Written independently of the oracle's version.
__host__ __device__ __forceinline__ int64_t position(int32_t dir, int64_t L, int32_t H, int32_t W,
                                                     int64_t t)
{
    if (dir == SS_DIR_FWD)
        return t;
    if (dir == SS_DIR_REV)
        return L - 1 - t;
    const int64_t s = (dir == SS_DIR_COL_REV) ? (L - 1 - t) : t;  // column-major step index
    const int64_t col = s / H;
    const int64_t row = s - col * H;
    return row * W + col;
}

// ---------------------------------------------------------------------------- shared layout

template <typename io_t, int NS, int WARPS, bool GATE, bool PHASE1>
struct Layout {
    static constexpr int DC = 32 * WARPS;                           // channels per CTA
    static constexpr int ROW = DC * (int)sizeof(io_t);               // bytes of one row slice
    static constexpr int ROWS = kTile * ROW;                         // bytes of one tensor tile
    static constexpr int BCRAW = ((kTile * NS * (int)sizeof(io_t) + 32 + 15) / 16) * 16;
    static constexpr bool HAS_Z = GATE && !PHASE1;
    static constexpr bool HAS_C = !PHASE1;
    static constexpr int OFF_U = 0;
    static constexpr int OFF_DL = OFF_U + ROWS;
    static constexpr int OFF_Z = OFF_DL + ROWS;
    static constexpr int OFF_BR = OFF_Z + (HAS_Z ? ROWS : 0);
    static constexpr int OFF_CR = OFF_BR + BCRAW;
    static constexpr int OFF_POS = OFF_CR + (HAS_C ? BCRAW : 0);
    static constexpr int STAGE = ((OFF_POS + kTile * 4 + 127) / 128) * 128;
    static constexpr int OFF_BC = kStages * STAGE;                   // fp32 B (and C), 2 buffers
    static constexpr int BC_ONE = kTile * NS * 4;
    static constexpr int BC_BUF = BC_ONE * (HAS_C ? 2 : 1);
    static constexpr int OFF_BAR = OFF_BC + 2 * BC_BUF;
    static constexpr int OFF_FLAG = OFF_BAR + kStages * 8;
    static constexpr int BYTES = OFF_FLAG + 16;
    static_assert(ROW % 16 == 0 && BCRAW % 16 == 0 && OFF_POS % 16 == 0, "TMA destinations");
    static_assert(OFF_BAR % 8 == 0, "mbarrier alignment");
};

// ---------------------------------------------------------------------------- the scan kernel

template <typename io_t, int NS, int WARPS, bool GATE, bool PHASE1>
__global__ void __launch_bounds__(32 * WARPS)
    scan_kernel(const __grid_constant__ ScanParams p)
{
    using Lay = Layout<io_t, NS, WARPS, GATE, PHASE1>;
    constexpr int DC = Lay::DC;
    constexpr int NT = 32 * WARPS;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
    volatile int& s_abort = *reinterpret_cast<int*>(smem + Lay::OFF_FLAG);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;

    // ---- which (direction, batch row, segment, channel tile) this CTA owns
    const int64_t ntiles = (p.D + DC - 1) / DC;
    const int nseg = PHASE1 ? (p.S - 1) : p.S;
    int64_t blk = blockIdx.x;
    const int64_t tile = blk % ntiles;
    blk /= ntiles;
    const int seg = static_cast<int>(blk % nseg);
    blk /= nseg;
    const int64_t b = blk % p.batch;
    const int k = static_cast<int>(blk / p.batch);
    const int dir = p.dirs[k];

    const int64_t d0 = tile * DC;
    const int dcv = static_cast<int>((p.D - d0) < DC ? (p.D - d0) : DC);  // valid channels
    const int64_t d = d0 + tid;
    const bool active = tid < dcv;
    const int64_t t_begin = static_cast<int64_t>(seg) * p.seg_len;
    const int64_t t_end = (t_begin + p.seg_len < p.L) ? (t_begin + p.seg_len) : p.L;
    const int64_t ntile_t = (t_end - t_begin + kTile - 1) / kTile;

    const int esz = static_cast<int>(sizeof(io_t));
    const uint32_t row_bytes = static_cast<uint32_t>(dcv) * esz;

    const io_t* gu = static_cast<const io_t*>(p.u);
    const io_t* gz = static_cast<const io_t*>(p.z);
    const io_t* gdl = static_cast<const io_t*>(p.delta);
    const io_t* gB = static_cast<const io_t*>(p.B);
    const io_t* gC = static_cast<const io_t*>(p.C);
    const int64_t kb = static_cast<int64_t>(k) * p.batch + b;  // (direction, batch) row block

    if (tid == 0) {
        s_abort = 0;
        for (int s = 0; s < kStages; ++s)
            mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();

    // B/C tiles are copied from a 16-byte aligned superset of their rows; this is the offset of
    // the first wanted element inside the copied block.
    auto bc_src = [&](const io_t* base, int64_t t0, int rows, uint32_t& bytes, int& skip) {
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(base + (kb * p.L + t0) * p.N);
        const uintptr_t a1 = reinterpret_cast<uintptr_t>(base + (kb * p.L + t0 + rows) * p.N);
        const uintptr_t lo = a0 & ~static_cast<uintptr_t>(15);
        const uintptr_t hi = (a1 + 15) & ~static_cast<uintptr_t>(15);
        bytes = static_cast<uint32_t>(hi - lo);
        skip = static_cast<int>((a0 - lo) / sizeof(io_t));
        return reinterpret_cast<const void*>(lo);
    };

    // Fill stage `st` with time tile `it` (warp 0 only; all 32 lanes issue copies).
    auto issue = [&](int64_t it, int st) {
        unsigned char* sb = smem + st * Lay::STAGE;
        const int64_t t0 = t_begin + it * kTile;
        const int rows = static_cast<int>((t_end - t0) < kTile ? (t_end - t0) : kTile);
        uint32_t bbytes, cbytes = 0;
        int bskip, cskip;
        const void* bsrc = bc_src(gB, t0, rows, bbytes, bskip);
        const void* csrc = Lay::HAS_C ? bc_src(gC, t0, rows, cbytes, cskip) : nullptr;
        if (lane == 0) {
            const uint32_t tx = static_cast<uint32_t>(rows) * row_bytes * (Lay::HAS_Z ? 3u : 2u) +
                                bbytes + cbytes;
            mbar_expect_tx(&full[st], tx);
        }
        __syncwarp();
        int32_t* pos = reinterpret_cast<int32_t*>(sb + Lay::OFF_POS);
        for (int r = lane; r < rows; r += 32) {
            const int64_t t = t0 + r;
            const int64_t pp = position(dir, p.L, p.H, p.W, t);
            pos[r] = static_cast<int32_t>(pp);
            bulk_g2s(sb + Lay::OFF_U + r * Lay::ROW, gu + (b * p.L + pp) * p.D + d0, row_bytes,
                     &full[st]);
            bulk_g2s(sb + Lay::OFF_DL + r * Lay::ROW, gdl + (kb * p.L + t) * p.D + d0, row_bytes,
                     &full[st]);
            if (Lay::HAS_Z)
                bulk_g2s(sb + Lay::OFF_Z + r * Lay::ROW, gz + (b * p.L + pp) * p.D + d0, row_bytes,
                         &full[st]);
        }
        if (lane == 0) {
            bulk_g2s(sb + Lay::OFF_BR, bsrc, bbytes, &full[st]);
            if (Lay::HAS_C)
                bulk_g2s(sb + Lay::OFF_CR, csrc, cbytes, &full[st]);
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&full[st]);
    };

    // ---- per-channel constants
    float a_l[NS];       // A[d, n] (natural units; multiplies Delta*log2(e))
    bool chain = true;   // A[d, n] == (n+1) * A[d, 0] for all n
    float dskip = 0.f, bias2 = 0.f;
    if (active) {
#pragma unroll
        for (int n = 0; n < NS; ++n) {
            a_l[n] = (n < p.N) ? p.A[d * p.N + n] : 0.f;
            if (n < p.N && a_l[n] != static_cast<float>(n + 1) * a_l[0])
                chain = false;
        }
        dskip = p.Dskip ? p.Dskip[d] : 0.f;
        bias2 = (p.bias ? p.bias[d] : 0.f) * kLog2e;
    } else {
#pragma unroll
        for (int n = 0; n < NS; ++n)
            a_l[n] = 0.f;
    }
    const bool use_chain = __all_sync(0xffffffffu, chain) && !p.force_generic;

    // ---- state: normalised k = h / w_prev
    float kst[NS];
    float wprev = 1.f;
#pragma unroll
    for (int n = 0; n < NS; ++n)
        kst[n] = 0.f;
    if (!PHASE1 && seg > 0 && active) {
        // fold the carries of segments 0..seg-1: h <- exp(A * sumDelta_s) * h + h_s
        for (int s = 0; s < seg; ++s) {
            const int64_t ci = (kb * p.S + s) * p.D + d;
            const float sd = p.carry_s[ci];
            const float* ch = p.carry_h + ci * p.N;
#pragma unroll
            for (int n = 0; n < NS; ++n)
                if (n < p.N)
                    kst[n] = ex2(a_l[n] * sd) * kst[n] + ch[n];
        }
    }
    float dsum = 0.f;  // sum of Delta*log2(e) over this segment (aggregate launch)

    // ---- prologue: fill kStages-1 stages
    int64_t issued = 0;
    if (warp == 0) {
        for (; issued < kStages - 1 && issued < ntile_t; ++issued)
            issue(issued, static_cast<int>(issued % kStages));
    }

    float* bcbuf = reinterpret_cast<float*>(smem + Lay::OFF_BC);
    int64_t failed_at = -1;
    for (int64_t it = 0; it < ntile_t; ++it) {
        const int st = static_cast<int>(it % kStages);
        const uint32_t parity = static_cast<uint32_t>((it / kStages) & 1);
        unsigned char* sb = smem + st * Lay::STAGE;
        const int64_t t0 = t_begin + it * kTile;
        const int rows = static_cast<int>((t_end - t0) < kTile ? (t_end - t0) : kTile);

        if (!mbar_wait_bounded(&full[st], parity, kWaitLimitNs)) {
            atomicOr(&g_ss_status, kStatusTimeout);
            s_abort = 1;
        }
        // convert this tile's B (and C) to fp32; B carries the ln 2 of w = Delta*u
        float* bf = bcbuf + (it & 1) * (Lay::BC_BUF / 4);
        {
            uint32_t bbytes, cbytes = 0;
            int bskip = 0, cskip = 0;
            bc_src(gB, t0, rows, bbytes, bskip);
            if (Lay::HAS_C)
                bc_src(gC, t0, rows, cbytes, cskip);
            const io_t* br = reinterpret_cast<const io_t*>(sb + Lay::OFF_BR) + bskip;
            const io_t* cr = reinterpret_cast<const io_t*>(sb + Lay::OFF_CR) + cskip;
            for (int idx = tid; idx < kTile * NS; idx += NT) {
                const int r = idx / NS, n = idx - (idx / NS) * NS;
                const bool ok = r < rows && n < p.N;
                bf[idx] = ok ? Io<io_t>::ld(br + r * p.N + n) * kLn2 : 0.f;
                if (Lay::HAS_C)
                    bf[kTile * NS + idx] = ok ? Io<io_t>::ld(cr + r * p.N + n) : 0.f;
            }
        }
        __syncthreads();  // tile `it` converted; every thread is done with tile it-1
        if (s_abort) {
            failed_at = it;
            break;
        }
        if (warp == 0 && issued < ntile_t) {
            issue(issued, static_cast<int>(issued % kStages));
            ++issued;
        }

        if (active) {
            const io_t* su = reinterpret_cast<const io_t*>(sb + Lay::OFF_U);
            const io_t* sdl = reinterpret_cast<const io_t*>(sb + Lay::OFF_DL);
            const io_t* sz = reinterpret_cast<const io_t*>(sb + Lay::OFF_Z);
            const int32_t* pos = reinterpret_cast<const int32_t*>(sb + Lay::OFF_POS);
            const float4* B4 = reinterpret_cast<const float4*>(bf);
            const float4* C4 = reinterpret_cast<const float4*>(bf + kTile * NS);
            for (int r = 0; r < rows; ++r) {
                const float uv = Io<io_t>::ld(su + r * DC + tid);
                const float dr = Io<io_t>::ld(sdl + r * DC + tid);
                // x = (delta + bias) * log2(e); Delta*log2(e) = softplus in base 2 of x
                const float x = fmaf(dr, kLog2e, bias2);
                float sp2 = x;
                if (p.softplus) {
                    const float e = ex2(-fabsf(x));              // 2^-|x| in (0, 1]
                    const float l_big = lg2(1.f + e);
                    // log2(1+e) for small e: e*log2(e)*(1 - e/2), relative error < e^2/3
                    const float l_small = e * fmaf(e, -0.5f * kLog2e, kLog2e);
                    sp2 = fmaxf(x, 0.f) + (e < 0.00390625f ? l_small : l_big);
                }
                float w = sp2 * uv;                               // = Delta*u / ln 2
                w = fabsf(w) < kTinyW ? kTinyW : w;
                const float rr = wprev * rcp(w);
                wprev = w;
                if (PHASE1)
                    dsum += sp2;
                float yp = 0.f;
                if (use_chain) {
                    const float q = ex2(sp2 * a_l[0]);
                    float c = rr;
#pragma unroll
                    for (int n4 = 0; n4 < NS / 4; ++n4) {
                        const float4 bq = B4[r * (NS / 4) + n4];
                        const float bv[4] = {bq.x, bq.y, bq.z, bq.w};
                        float cv[4] = {0.f, 0.f, 0.f, 0.f};
                        if (!PHASE1) {
                            const float4 cq = C4[r * (NS / 4) + n4];
                            cv[0] = cq.x; cv[1] = cq.y; cv[2] = cq.z; cv[3] = cq.w;
                        }
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            c *= q;
                            kst[n4 * 4 + j] = fmaf(c, kst[n4 * 4 + j], bv[j]);
                            if (!PHASE1)
                                yp = fmaf(cv[j], kst[n4 * 4 + j], yp);
                        }
                    }
                } else {
#pragma unroll
                    for (int n4 = 0; n4 < NS / 4; ++n4) {
                        const float4 bq = B4[r * (NS / 4) + n4];
                        const float bv[4] = {bq.x, bq.y, bq.z, bq.w};
                        float cv[4] = {0.f, 0.f, 0.f, 0.f};
                        if (!PHASE1) {
                            const float4 cq = C4[r * (NS / 4) + n4];
                            cv[0] = cq.x; cv[1] = cq.y; cv[2] = cq.z; cv[3] = cq.w;
                        }
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float c = rr * ex2(sp2 * a_l[n4 * 4 + j]);
                            kst[n4 * 4 + j] = fmaf(c, kst[n4 * 4 + j], bv[j]);
                            if (!PHASE1)
                                yp = fmaf(cv[j], kst[n4 * 4 + j], yp);
                        }
                    }
                }
                if (!PHASE1) {
                    float y = fmaf(dskip, uv, w * yp);
                    const int64_t pp = pos[r];
                    if (p.ypart) {
                        p.ypart[(kb * p.L + pp) * p.D + d] = y;
                    } else {
                        if (GATE) {
                            const float zv = Io<io_t>::ld(sz + r * DC + tid);
                            y *= zv * rcp(1.f + ex2(-zv * kLog2e));
                        }
                        static_cast<io_t*>(p.out)[(b * p.L + pp) * p.D + d] = Io<io_t>::st(y);
                    }
                }
            }
        }
    }

    if (failed_at >= 0) {
        // let the copies this CTA still has in flight (tiles failed_at .. issued-1) land before
        // its shared memory goes away; each wait is bounded as well
        if (warp == 0 && lane == 0) {
            for (int64_t j = failed_at; j < issued; ++j)
                (void)mbar_wait_bounded(&full[j % kStages], static_cast<uint32_t>((j / kStages) & 1),
                                        kWaitLimitNs / 4);
        }
        __syncthreads();
        return;
    }

    if (!active)
        return;
    if (PHASE1) {
        const int64_t ci = (kb * p.S + seg) * p.D + d;
        p.carry_s[ci] = dsum;
#pragma unroll
        for (int n = 0; n < NS; ++n)
            if (n < p.N)
                p.carry_h[ci * p.N + n] = wprev * kst[n];
    } else if (p.last_state && seg == p.S - 1) {
        float* ls = p.last_state + (kb * p.D + d) * p.N;
#pragma unroll
        for (int n = 0; n < NS; ++n)
            if (n < p.N)
                ls[n] = wprev * kst[n];
    }
}

// ---------------------------------------------------------------------------- merge kernel

template <typename io_t, bool GATE>
__global__ void __launch_bounds__(256) merge_kernel(const __grid_constant__ MergeParams p)
{
    const int64_t total = p.rows * p.D;
    const int64_t plane = total;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float y = 0.f;
        for (int k = 0; k < p.K; ++k)
            y += p.ypart[k * plane + i];
        if (GATE) {
            const float zv = Io<io_t>::ld(static_cast<const io_t*>(p.z) + i);
            y *= zv * rcp(1.f + ex2(-zv * kLog2e));
        }
        static_cast<io_t*>(p.out)[i] = Io<io_t>::st(y);
    }
}

// ---------------------------------------------------------------------------- dispatch

constexpr int kWarps = 2;

template <typename io_t, int NS, bool GATE, bool PHASE1>
cudaError_t launch_t(const ScanParams& p, cudaStream_t stream)
{
    using Lay = Layout<io_t, NS, kWarps, GATE, PHASE1>;
    auto kern = scan_kernel<io_t, NS, kWarps, GATE, PHASE1>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::BYTES);
    if (e != cudaSuccess)
        return e;
    const int64_t ntiles = (p.D + Lay::DC - 1) / Lay::DC;
    const int64_t nseg = PHASE1 ? (p.S - 1) : p.S;
    const int64_t nblocks = ntiles * nseg * p.batch * p.K;
    if (nblocks <= 0)
        return cudaSuccess;
    kern<<<static_cast<unsigned int>(nblocks), 32 * kWarps, Lay::BYTES, stream>>>(p);
    return cudaGetLastError();
}

template <typename io_t, int NS>
cudaError_t launch_ns(const ScanParams& p, int phase1, cudaStream_t stream)
{
    const bool gate = p.z != nullptr && p.ypart == nullptr;
    if (phase1)
        return launch_t<io_t, NS, false, true>(p, stream);
    return gate ? launch_t<io_t, NS, true, false>(p, stream)
                : launch_t<io_t, NS, false, false>(p, stream);
}

template <typename io_t>
cudaError_t launch_io(const ScanParams& p, int phase1, cudaStream_t stream)
{
    if (p.N <= 4)
        return launch_ns<io_t, 4>(p, phase1, stream);
    if (p.N <= 8)
        return launch_ns<io_t, 8>(p, phase1, stream);
    return launch_ns<io_t, 16>(p, phase1, stream);
}

}  // namespace

int channels_per_cta() { return 32 * kWarps; }

cudaError_t launch_scan(const ScanParams& p, int io_dtype, int phase1, cudaStream_t stream)
{
    return io_dtype == SS_BF16 ? launch_io<__nv_bfloat16>(p, phase1, stream)
                               : launch_io<float>(p, phase1, stream);
}

cudaError_t launch_merge(const MergeParams& p, int io_dtype, cudaStream_t stream)
{
    const int64_t total = p.rows * p.D;
    if (total <= 0)
        return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (total + 255) / 256;
    if (blocks > static_cast<int64_t>(sms) * 16)
        blocks = static_cast<int64_t>(sms) * 16;
    const bool gate = p.z != nullptr;
    if (io_dtype == SS_BF16) {
        if (gate)
            merge_kernel<__nv_bfloat16, true><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
        else
            merge_kernel<__nv_bfloat16, false><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
    } else {
        if (gate)
            merge_kernel<float, true><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
        else
            merge_kernel<float, false><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
    }
    return cudaGetLastError();
}

int64_t position_host(int32_t dir, int64_t L, int32_t H, int32_t W, int64_t t)
{
    return position(dir, L, H, W, t);
}

cudaError_t read_status(cudaStream_t stream, bool clear, unsigned int* value)
{
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess)
        return e;
    e = cudaMemcpyFromSymbol(value, g_ss_status, sizeof(unsigned int));
    if (e != cudaSuccess || !clear)
        return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_ss_status, &zero, sizeof(unsigned int));
}

}  // namespace ss
