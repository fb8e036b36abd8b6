// Selective scan (S6) forward kernels for sm_100a.
//
// One thread owns one channel d of one (batch row, direction, segment) and keeps that channel's
// N-state vector in registers for the whole segment ("Understanding Mamba from zero" sec. 5:
// per channel and per state the recurrence is the scalar affine map h_t = a_t h_{t-1} + b_t).
// A CTA of 32*WARPS threads owns a tile of adjacent channels.  Its inputs stream through a
// ring of 4-5 shared-memory stages of kTile steps each, filled by asynchronous bulk copies
// that complete on mbarriers: one tensor-map box (cp.async.bulk.tensor) per tile for u, z and
// delta (rows picked through the direction's index map: a 2D box for the row orders, 3D boxes
// of 8 image rows for the column orders, one bulk copy per row otherwise), plus one bulk copy
// each for the B and C tiles, which every channel of the CTA shares.  The producer duty
// (refilling the ring, converting B and C to the state type once per tile) rotates over the warps.
// Everything of a step -- the optional causal convolution of u, softplus, exp, the recurrence,
// the C readout, the D skip and the silu gate -- happens in registers; each input element is
// read from HBM once and each output element written once.
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
//  of w = Delta*u is folded into the fp32 copy of B.  fp32 inputs (and the exact-ZOH Bbar) take
//  a precise path instead: h = expm1(Delta*A)*h + (h + Bbar*u*B), with expm1 from a Taylor
//  polynomial near zero (so Abar is never rounded to fp32) and softplus from an atanh series.
//  With fp32 inputs that path keeps the state, the C readout and the segment carries in fp64
//  (B200 runs fp64 at half the fp32 rate): an fp32 state loses about one rounding of |h| per
//  step, which over thousands of steps of a slowly decaying state reaches the 1e-4 relative bar
//  at near-zero outputs; in fp64 the error is that of the fp32 per-step factors (Delta, expm1),
//  which does not accumulate.
//
// Long sequences are split into S segments (the chunked scan of "S4 -> Mamba" sec. 2.2): a
// first launch scans segments 0..S-2 from a zero state and stores each end state and the
// segment's sum of Delta; the second launch starts segment s from the carry obtained by
// folding the carries of segments 0..s-1 with the affine combine (P2, h2) o (P1, h1) =
// (P2*P1, P2*h1 + h2), P = exp(A * sum Delta).
//
// Options: an initial state, the exact ZOH Bbar, a causal depthwise convolution + SiLU of u per
// direction, int8 delta codes with per-channel scales, an input and/or a parameter set per
// direction (see include/selective_scan.h).
//
// Every wait on an mbarrier is bounded in time.  A wait that gives up sets the library's device
// error word (read by selective_scan_device_status), waits a bounded time for the copies this
// CTA still has in flight, and the whole CTA returns.
//
// This header holds the kernel, the direction merge and their launch templates; ss_scan_f32.cu,
// ss_scan_bf16.cu and ss_scan_bf16_i8.cu instantiate them per io type and delta storage
// (compiled in parallel), and ss_scan.cu holds the host dispatch.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "ss_internal.h"
#include "ss_device.cuh"

namespace ss {

namespace {

// log(1 + e) for e in [0, 1], relative error ~1e-7: 2*atanh(s) with s = e / (2 + e) <= 1/3,
// odd series up to s^15 (truncation < 2e-9 relative).
__device__ __forceinline__ float log1p_unit(float e)
{
    const float s = e * rcp(2.f + e);
    const float s2 = s * s;
    float p = 2.f / 15.f;
    p = fmaf(p, s2, 2.f / 13.f);
    p = fmaf(p, s2, 2.f / 11.f);
    p = fmaf(p, s2, 2.f / 9.f);
    p = fmaf(p, s2, 2.f / 7.f);
    p = fmaf(p, s2, 2.f / 5.f);
    p = fmaf(p, s2, 2.f / 3.f);
    p = fmaf(p, s2, 2.f);
    return s * p;
}

// exp(x) - 1 with relative accuracy ~1e-7 near 0 (Taylor to x^8 for |x| <= 0.35, truncation
// < 3e-10 relative), exp through ex2 elsewhere.
__device__ __forceinline__ float expm1_acc(float x)
{
    float p = 1.f / 40320.f;
    p = fmaf(p, x, 1.f / 5040.f);
    p = fmaf(p, x, 1.f / 720.f);
    p = fmaf(p, x, 1.f / 120.f);
    p = fmaf(p, x, 1.f / 24.f);
    p = fmaf(p, x, 1.f / 6.f);
    p = fmaf(p, x, 0.5f);
    p = fmaf(p, x, 1.f);
    const float small = x * p;
    const float big = ex2(x * 1.4426950408889634f) - 1.f;
    return fabsf(x) <= 0.35f ? small : big;
}

// ---------------------------------------------------------------------------- element types

template <typename T> struct Io;
template <> struct Io<int8_t> {  // int8 Delta codes (loaded only)
    static __device__ __forceinline__ float ld(const int8_t* p) { return static_cast<float>(*p); }
};
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

// ---------------------------------------------------------------------------- shared layout

// One pipeline stage holds kTile rows of u, delta and z for the CTA's channels (as copied),
// the raw B and C tiles, their copies in the state type, and the output row offsets of the tile.
template <typename io_t, typename dl_t, int NS, int WARPS, bool GATE, bool PHASE1, int STAGES>
struct Layout {
    static constexpr int DC = 32 * WARPS;                           // channels per CTA
    static constexpr int ROW = DC * (int)sizeof(io_t);               // bytes of one row slice
    static constexpr int ROWS = kTile * ROW;                         // bytes of one tensor tile
    static constexpr int ROWS_DL = kTile * DC * (int)sizeof(dl_t);   // bytes of one delta tile
    static constexpr int BCRAW = ((kTile * NS * (int)sizeof(io_t) + 32 + 15) / 16) * 16;
    static constexpr bool HAS_Z = GATE && !PHASE1;
    static constexpr bool HAS_C = !PHASE1;
    // each field is an array over the stages; tile fields come first (128-byte aligned for the
    // tensor copies), the rest is packed at 16-byte alignment to keep the CTA's footprint small
    static constexpr int OFF_U = 0;
    static constexpr int OFF_DL = OFF_U + STAGES * ROWS;
    static constexpr int OFF_Z = OFF_DL + STAGES * ROWS_DL;
    static constexpr int OFF_BR = OFF_Z + (HAS_Z ? STAGES * ROWS : 0);
    static constexpr int OFF_CR = OFF_BR + STAGES * BCRAW;
    // B, then C, converted to the state type (fp64 for fp32 io, else fp32)
    static constexpr int OFF_BF = OFF_CR + (HAS_C ? STAGES * BCRAW : 0);
    static constexpr int BF_ONE = kTile * NS * (std::is_same<io_t, float>::value ? 8 : 4);
    static constexpr int BF_STRIDE = BF_ONE * (HAS_C ? 2 : 1);
    static constexpr int OFF_OUT = OFF_BF + STAGES * BF_STRIDE;           // int32 row offsets
    static constexpr int OUT_STRIDE = kTile * 4;
    static constexpr int OFF_BAR = OFF_OUT + STAGES * OUT_STRIDE;         // full, ready, empty
    static constexpr int OFF_FLAG = OFF_BAR + 3 * STAGES * 8;
    static constexpr int BYTES = OFF_FLAG + 16;
    static_assert(ROWS % 128 == 0 && ROWS_DL % 128 == 0 && BCRAW % 16 == 0 && OFF_BR % 128 == 0 && OFF_BF % 16 == 0 &&
                      BF_STRIDE % 16 == 0 && OFF_OUT % 8 == 0,
                  "tensor-copy destinations need 128-byte and vector accesses 16-byte alignment");
};

// ---------------------------------------------------------------------------- the scan kernel
//
// Pipeline of one CTA (WARPS warps, every warp scans; in iteration it, warp it % WARPS also
// produces):
//   full[s]  completes when the bulk copies of the tile in stage s have landed (tx count);
//   ready[s] completes when the producing warp has converted that tile's B and C to the
//            state type (fp32, or fp64 for fp32 io);
//   empty[s] completes when all WARPS warps are done with the tile in stage s.
// The producer of iteration it converts tile it+1 (whose copies were issued earlier) and
// refills the stage released by tile it-2 with tile it+kStages-2, so kStages-2 tiles are in
// flight ahead of the one being scanned; only the producer ever waits on another warp (for the
// stage it refills), so the pipeline cannot deadlock.

template <typename io_t, typename dl_t, int NS, int WARPS, bool GATE, bool PHASE1, bool YPART,
          bool CONV>
__global__ void __launch_bounds__(32 * WARPS, PHASE1 ? 8 : 6)
    scan_kernel(const __grid_constant__ ScanParams p)
{
    // Scans that write per-direction partial outputs (several directions, short sequences,
    // column-order boxes) keep one more tile in flight; the others keep the ring smaller so
    // that more CTAs fit on an SM (both measured on B200).
    constexpr int kStages = YPART ? 5 : 4;
    using Lay = Layout<io_t, dl_t, NS, WARPS, GATE, PHASE1, kStages>;
    // int8 Delta codes: delta_raw = code * delta_scale[d]
    constexpr bool DQ = std::is_same<dl_t, int8_t>::value;
    // the producer refills the stage released two tiles back and prepares the next tile, so at
    // least four stages are needed for a tile to be in flight while the current one is scanned
    static_assert(kStages >= 4, "the pipeline needs at least four stages");
    // fp32 inputs take the precise arithmetic, bf16 inputs the fast one
    constexpr bool PRECISE = sizeof(io_t) == 4;
    // the precise arithmetic also serves the exact-ZOH Bbar for any io type
    const bool precise = PRECISE || p.zoh != 0;
    // fp32 io: fp64 state, readout and segment carries (the precise arithmetic only)
    constexpr bool WIDE = std::is_same<io_t, float>::value;
    using st_t = typename std::conditional<WIDE, double, float>::type;
    st_t* const carry_h = reinterpret_cast<st_t*>(p.carry_h);
    st_t* const carry_s = reinterpret_cast<st_t*>(p.carry_s);
    constexpr int DC = Lay::DC;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
    uint64_t* ready = full + kStages;
    uint64_t* empty = ready + kStages;
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + Lay::OFF_FLAG);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;

    // ---- which (segment, direction, batch row, channel tile) this CTA owns; segments are the
    // slowest index, so the first CTAs of a scan launch are the segment-0 ones, which need no
    // carry and can run while the segment aggregates are still being computed
    const int64_t ntiles = (p.D + DC - 1) / DC;
    const int64_t per_seg = ntiles * p.batch * p.K;
    int64_t blk = blockIdx.x;
    const int seg = static_cast<int>(blk / per_seg);
    blk -= static_cast<int64_t>(seg) * per_seg;
    const int64_t tile = blk % ntiles;
    blk /= ntiles;
    const int64_t b = blk % p.batch;
    const int k = static_cast<int>(blk / p.batch);
    // constant indices keep the parameter array out of local memory
    const int dir = k == 0 ? p.dirs[0] : k == 1 ? p.dirs[1] : k == 2 ? p.dirs[2] : p.dirs[3];

    const int64_t d0 = tile * DC;
    const int dcv = static_cast<int>((p.D - d0) < DC ? (p.D - d0) : DC);  // valid channels
    const int64_t d = d0 + tid;
    const bool active = tid < dcv;
    const int64_t t_begin = static_cast<int64_t>(seg) * p.seg_len;
    const int64_t t_end = (t_begin + p.seg_len < p.L) ? (t_begin + p.seg_len) : p.L;
    const int64_t ntile_t = (t_end - t_begin + kTile - 1) / kTile;

    const uint32_t row_bytes = static_cast<uint32_t>(dcv) * static_cast<uint32_t>(sizeof(io_t));
    const io_t* gu = static_cast<const io_t*>(p.u);
    const io_t* gz = static_cast<const io_t*>(p.z);
    const io_t* gB = static_cast<const io_t*>(p.B);
    const io_t* gC = static_cast<const io_t*>(p.C);
    const int64_t kb = static_cast<int64_t>(k) * p.batch + b;  // (direction, batch) row block
    const int64_t ub = p.u_per_dir ? kb : b;                   // row block of this CTA's u
    // output rows: out[b, p, :] for one direction, ypart[k, b, p, :] for several; a row's
    // element offset from this CTA's base (row 0 of its block, channel d0) fits in 32 bits
    const int64_t out_base = (p.ypart ? kb * p.L : b * p.L) * p.D + d0;

    if (tid == 0) {
        *s_abort = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&ready[s], 1);
            mbar_init(&empty[s], WARPS);
        }
        fence_mbar_init();
    }
    __syncthreads();
    // the next launch (the scan after the aggregates, the merge after the scan) may start now;
    // it waits for this grid's results itself where it needs them
    pdl_launch_dependents();
    if (p.test_timeout) {
        // failure-detection test hook: nobody arrives on ready[0], so this bounded wait gives
        // up; no copy has been issued yet, so the CTA can return at once
        if (!mbar_wait_bounded(&ready[0], 0, kTestWaitNs) && tid == 0)
            atomicOr(p.status, kStatusTimeout);
        return;
    }

    // B/C tiles are copied from a 16-byte aligned superset of their rows; `skip` is the offset
    // (in elements) of the first wanted element inside the copied block.  With whole 16-byte
    // rows (N * element size a multiple of 16) every tile starts aligned and `skip` is 0.
    const bool bc_whole = (p.N * sizeof(io_t)) % 16 == 0;
    auto bc_src = [&](const io_t* base, int64_t it, int rows, uint32_t& bytes, int& skip) {
        const int64_t t0 = t_begin + it * kTile;
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(base + (kb * p.L + t0) * p.N);
        const uintptr_t a1 = reinterpret_cast<uintptr_t>(base + (kb * p.L + t0 + rows) * p.N);
        const uintptr_t lo = a0 & ~static_cast<uintptr_t>(15);
        const uintptr_t hi = (a1 + 15) & ~static_cast<uintptr_t>(15);
        bytes = static_cast<uint32_t>(hi - lo);
        skip = static_cast<int>((a0 - lo) / sizeof(io_t));
        return reinterpret_cast<const void*>(lo);
    };
    auto tile_rows = [&](int64_t it) {
        const int64_t t0 = t_begin + it * kTile;
        return static_cast<int>((t_end - t0) < kTile ? (t_end - t0) : kTile);
    };

    // How u and z rows reach shared memory: 0 = one box of kTile spatial rows (forward and
    // reverse orders visit contiguous rows), 1 = boxes of 8 rows of one image column (column
    // orders, H % 8 == 0), 2 = one bulk copy per row.  Step t0 + r of a tile reads u/z row
    // (r ^ xmask) of the stage; delta rows are always in scan order.
    const int umode = (dir == SS_DIR_FWD || dir == SS_DIR_REV) ? 0 : (p.col3d ? 1 : 2);
    const int xmask =
        dir == SS_DIR_REV ? (kTile - 1) : (dir == SS_DIR_COL_REV && umode == 1 ? 7 : 0);
    constexpr uint32_t kBox2 = static_cast<uint32_t>(DC) * kTile * sizeof(io_t);
    constexpr uint32_t kBoxDL = static_cast<uint32_t>(DC) * kTile * sizeof(dl_t);
    constexpr uint32_t kBox3 = static_cast<uint32_t>(DC) * 8 * sizeof(io_t);
    constexpr uint32_t kUZ = Lay::HAS_Z ? 2u : 1u;

    // Fill stage st with time tile `it` (called by the producing warp).
    auto issue = [&](int64_t it, int st) {
        const int64_t t0 = t_begin + it * kTile;
        const int rows = tile_rows(it);
        uint32_t bbytes, cbytes = 0;
        int bskip, cskip;
        const void* bsrc = bc_src(gB, it, rows, bbytes, bskip);
        const void* csrc = Lay::HAS_C ? bc_src(gC, it, rows, cbytes, cskip) : nullptr;
        if (lane == 0) {
            uint32_t tx = kBoxDL + bbytes + cbytes;  // delta box, B, C
            if (umode == 0)
                tx += kUZ * kBox2;
            else if (umode == 1)
                tx += kUZ * kBox3 * static_cast<uint32_t>(rows / 8);
            else
                tx += kUZ * static_cast<uint32_t>(rows) * row_bytes;
            mbar_expect_tx(&full[st], tx);
            tma_2d(smem + Lay::OFF_DL + st * Lay::ROWS_DL, &p.tm_dl, static_cast<int32_t>(d0),
                   static_cast<int32_t>(kb * p.L + t0), &full[st]);
            if (umode == 0) {
                // reverse order: the box ends at the row of step t0
                const int64_t prow = (dir == SS_DIR_FWD ? t0 : p.L - t0 - kTile);
                tma_2d(smem + Lay::OFF_U + st * Lay::ROWS, &p.tm_u, static_cast<int32_t>(d0),
                       static_cast<int32_t>(ub * p.L + prow), &full[st]);
                if (Lay::HAS_Z)
                    tma_2d(smem + Lay::OFF_Z + st * Lay::ROWS, &p.tm_z, static_cast<int32_t>(d0),
                           static_cast<int32_t>(b * p.L + prow), &full[st]);
            } else if (umode == 1) {
                for (int sub = 0; sub < rows / 8; ++sub) {
                    const int64_t tt = t0 + 8 * sub;
                    // column-major index of the lowest image row of the box
                    const int64_t c = dir == SS_DIR_COL ? tt : (p.L - 8 - tt);
                    const int64_t j = c / p.H, i = c - (c / p.H) * p.H;
                    tma_3d(smem + Lay::OFF_U + st * Lay::ROWS + 8 * sub * Lay::ROW, &p.tm_u3,
                           static_cast<int32_t>(d0), static_cast<int32_t>(j),
                           static_cast<int32_t>(ub * p.H + i), &full[st]);
                    if (Lay::HAS_Z)
                        tma_3d(smem + Lay::OFF_Z + st * Lay::ROWS + 8 * sub * Lay::ROW, &p.tm_z3,
                               static_cast<int32_t>(d0), static_cast<int32_t>(j),
                               static_cast<int32_t>(b * p.H + i), &full[st]);
                }
            }
            bulk_g2s(smem + Lay::OFF_BR + st * Lay::BCRAW, bsrc, bbytes, &full[st]);
            if (Lay::HAS_C)
                bulk_g2s(smem + Lay::OFF_CR + st * Lay::BCRAW, csrc, cbytes, &full[st]);
        }
        __syncwarp();
        int32_t* orow = reinterpret_cast<int32_t*>(smem + Lay::OFF_OUT + st * Lay::OUT_STRIDE);
        for (int r = lane; r < rows; r += 32) {
            const int64_t pp = position(dir, p.L, p.H, p.W, t0 + r);
            // L * D < 2^31 (checked on the host): 32-bit arithmetic
            orow[r] = static_cast<int32_t>(pp) * static_cast<int32_t>(p.D);
            if (umode == 2) {
                bulk_g2s(smem + Lay::OFF_U + st * Lay::ROWS + r * Lay::ROW, gu + (ub * p.L + pp) * p.D + d0,
                         row_bytes, &full[st]);
                if (Lay::HAS_Z)
                    bulk_g2s(smem + Lay::OFF_Z + st * Lay::ROWS + r * Lay::ROW, gz + (b * p.L + pp) * p.D + d0,
                             row_bytes, &full[st]);
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&full[st]);
    };

    // Convert tile `it`'s B (and C) to the state type (producing warp).  On the fast path B
    // carries the ln 2 of w = Delta*u / ln 2.
    auto convert = [&](int64_t it, int st) {
        const int rows = tile_rows(it);
        uint32_t bytes;
        int bskip = 0, cskip = 0;
        if (!bc_whole) {
            bc_src(gB, it, rows, bytes, bskip);
            if (Lay::HAS_C)
                bc_src(gC, it, rows, bytes, cskip);
        }
        const io_t* br = reinterpret_cast<const io_t*>(smem + Lay::OFF_BR + st * Lay::BCRAW) + bskip;
        const io_t* cr = reinterpret_cast<const io_t*>(smem + Lay::OFF_CR + st * Lay::BCRAW) + cskip;
        st_t* bf = reinterpret_cast<st_t*>(smem + Lay::OFF_BF + st * Lay::BF_STRIDE);
        const float bscale = precise ? 1.f : kLn2;
        if (!WIDE && NS == 16 && p.N == 16 && sizeof(io_t) == 2 && bskip == 0 && cskip == 0) {
            // 16 bf16 rows of 16 values per tensor: lane l converts 8 values (16 bytes) of B and
            // 8 of C; rows past the tile's end become 0
            static_assert(kTile * 16 * 2 == 32 * 16, "one 16-byte chunk per lane and tensor");
            const int r = lane >> 1;
            const bool ok = r < rows;
            auto cvt8 = [&](const io_t* src, st_t* dst, float scale) {
                const uint4 w = *reinterpret_cast<const uint4*>(src + 8 * lane);
                const uint32_t v[4] = {w.x, w.y, w.z, w.w};
                float f[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    f[2 * i] = ok ? __uint_as_float(v[i] << 16) * scale : 0.f;
                    f[2 * i + 1] = ok ? __uint_as_float(v[i] & 0xffff0000u) * scale : 0.f;
                }
                float4* d4 = reinterpret_cast<float4*>(reinterpret_cast<float*>(dst) + 8 * lane);
                d4[0] = make_float4(f[0], f[1], f[2], f[3]);
                d4[1] = make_float4(f[4], f[5], f[6], f[7]);
            };
            cvt8(br, bf, bscale);
            if (Lay::HAS_C)
                cvt8(cr, bf + kTile * NS, 1.f);
            return;
        }
        for (int idx = lane; idx < kTile * NS; idx += 32) {
            const int r = idx / NS, n = idx - (idx / NS) * NS;
            const bool ok = r < rows && n < p.N;
            bf[idx] = ok ? static_cast<st_t>(Io<io_t>::ld(br + r * p.N + n) * bscale) : st_t(0);
            if (Lay::HAS_C)
                bf[kTile * NS + idx] = ok ? static_cast<st_t>(Io<io_t>::ld(cr + r * p.N + n)) : st_t(0);
        }
    };

    // ---- per-channel constants
    float a_l[NS];       // A[d, n] (natural units; multiplies Delta*log2(e))
    bool chain = true;   // A[d, n] == (n+1) * A[d, 0] for all n
    float dskip = 0.f, bias2 = 0.f, bias_raw = 0.f;
    float dscale = 1.f, dscale2 = kLog2e;  // int8 codes: scale[d], and scale[d] * log2(e)
    if (active) {
        // parameters of this direction (one set shared by all directions unless per direction)
        const int64_t pk = p.params_per_dir ? static_cast<int64_t>(k) : 0;
        const float* Ak = p.A + pk * p.D * p.N;
#pragma unroll
        for (int n = 0; n < NS; ++n) {
            a_l[n] = (n < p.N) ? Ak[d * p.N + n] : 0.f;
            if (n < p.N && a_l[n] != static_cast<float>(n + 1) * a_l[0])
                chain = false;
        }
        dskip = p.Dskip ? p.Dskip[pk * p.D + d] : 0.f;
        bias_raw = p.bias ? p.bias[pk * p.D + d] : 0.f;
        bias2 = bias_raw * kLog2e;
        if (DQ) {
            dscale = p.delta_scale[d];
            dscale2 = dscale * kLog2e;
        }
    } else {
#pragma unroll
        for (int n = 0; n < NS; ++n)
            a_l[n] = 0.f;
    }
    const bool use_chain = __all_sync(0xffffffffu, chain) && !p.force_generic;
    const bool softplus = p.softplus != 0;

    // ---- causal depthwise convolution along this direction's scan order (CONV): the taps and
    // bias halved (exact), right-aligned so that cw[3] multiplies the current step, and the
    // inputs of the three steps before the segment (zero before step 0), read once from global
    // memory
    float cw[4] = {0.f, 0.f, 0.f, 0.f};
    float cbias = 0.f;
    float xm1 = 0.f, xm2 = 0.f, xm3 = 0.f;  // inputs of steps t-1, t-2, t-3
    if (CONV && active) {
        const float* wk = p.conv_w + (static_cast<int64_t>(k) * p.D + d) * p.conv_width;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const int j = s - (4 - p.conv_width);
            if (j >= 0)
                cw[s] = 0.5f * wk[j];
        }
        cbias = p.conv_b ? 0.5f * p.conv_b[static_cast<int64_t>(k) * p.D + d] : 0.f;
        auto halo = [&](int64_t t) {
            return t >= 0 ? Io<io_t>::ld(gu + (ub * p.L + position(dir, p.L, p.H, p.W, t)) * p.D + d)
                          : 0.f;
        };
        xm1 = halo(t_begin - 1);
        xm2 = halo(t_begin - 2);
        xm3 = halo(t_begin - 3);
    }
    // u of the current step from its raw input: the convolution and SiLU with CONV, else as is.
    // With h = c/2 (the halved taps), silu(c) = c * sigmoid(c) = h + h * tanh(h): one MUFU
    // operation on the fast path; the precise path takes c * 1/(1 + 2^(-c log2 e)).
    auto conv_step = [&](float xv, auto accurate_tag) {
        if (!CONV)
            return xv;
        const float h = fmaf(cw[3], xv, fmaf(cw[2], xm1, fmaf(cw[1], xm2, fmaf(cw[0], xm3, cbias))));
        xm3 = xm2;
        xm2 = xm1;
        xm1 = xv;
        if (decltype(accurate_tag)::value) {
            const float c = h + h;
            return c * rcp(1.f + ex2(-c * kLog2e));
        }
        return fmaf(h, tanh_approx(h), h);
    };

    // ---- state, as pairs (n, n+1): the fast path keeps k = h / w_prev, the precise path h
    // (NS doubles with fp32 io)
    using pair_t = typename std::conditional<WIDE, double, float2>::type;
    pair_t kst2[WIDE ? NS : NS / 2];
    st_t* kst = reinterpret_cast<st_t*>(kst2);
    float wprev = 1.f;
#pragma unroll
    for (int n = 0; n < NS; ++n)
        kst[n] = st_t(0);
    if (!PHASE1 && active && p.init_state) {
        const float* h0 = p.init_state + (kb * p.D + d) * p.N;
#pragma unroll
        for (int n = 0; n < NS; ++n)
            if (n < p.N)
                kst[n] = h0[n];
    }
    if (!PHASE1 && seg > 0) {
        // the carries come from the aggregate launch just before this one
        pdl_wait();
    }
    if (!PHASE1 && seg > 0 && active) {
        // fold the carries of segments 0..seg-1: h <- exp(A * sumDelta_s) * h + h_s
        for (int s = 0; s < seg; ++s) {
            const int64_t ci = (kb * p.S + s) * p.D + d;
            const st_t sd = __ldcg(carry_s + ci);
            const st_t* ch = carry_h + ci * p.N;
#pragma unroll
            for (int n = 0; n < NS; ++n) {
                if (n < p.N) {
                    if constexpr (WIDE)  // sd = sum of Delta
                        kst[n] = exp(static_cast<double>(a_l[n]) * sd) * kst[n] + __ldcg(ch + n);
                    else                 // sd = sum of Delta*log2(e)
                        kst[n] = ex2(a_l[n] * sd) * kst[n] + __ldcg(ch + n);
                }
            }
        }
    }
    // sum over this segment of Delta*log2(e), or of Delta in fp64 with fp32 io (aggregate launch)
    st_t dsum = st_t(0);

    // ---- pipeline.  Producer duty rotates: in iteration `it`, warp it % WARPS converts the B/C
    // of tile it+1 (one tile ahead, so no warp waits for a conversion) and refills the stage
    // released by tile it-2 with tile it+kStages-2.  Warp 0 starts the pipeline.
    volatile int* s_issued = s_abort + 1;  // tiles issued so far (read only on the error path)
    bool failed = false;
    int64_t my_issued = 0;                 // tiles this warp has issued (error path)
    if (warp == 0) {
        int64_t j = 0;
        for (; j < kStages - 2 && j < ntile_t; ++j)
            issue(j, static_cast<int>(j));
        my_issued = j;
        if (lane == 0)
            *s_issued = static_cast<int>(j);
        if (!mbar_wait_bounded(&full[0], 0, kWaitLimitNs)) {
            failed = true;
        } else {
            convert(0, 0);
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&ready[0]);
        }
    }
    // stage st = it % kStages and phase parity ph = (it / kStages) & 1 of tile it, advanced at
    // the end of each iteration (no 64-bit division per tile)
    int st = 0;
    uint32_t ph = 0;
    for (int64_t it = 0; it < ntile_t && !failed;
         ++it, ph ^= (st == kStages - 1) ? 1u : 0u, st = (st == kStages - 1) ? 0 : st + 1) {
        const int rows = tile_rows(it);
        if (*s_abort) {
            failed = true;
            break;
        }
        if (warp == static_cast<int>(it % WARPS)) {
            const int64_t n1 = it + 1;
            // tile it+1: the next stage, in the next phase when it wraps
            const int st1 = (st == kStages - 1) ? 0 : st + 1;
            const uint32_t ph1 = ph ^ ((st == kStages - 1) ? 1u : 0u);
            if (n1 < ntile_t) {
                if (!mbar_wait_bounded(&full[st1], ph1, kWaitLimitNs)) {
                    failed = true;
                } else {
                    convert(n1, st1);
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&ready[st1]);
                }
            }
            // tile it+kStages-2 goes to the stage tile it-2 used; that stage's previous phase
            // (the release by tile it-2) has parity ((it + kStages - 2) / kStages - 1) & 1
            const int64_t nx = it + kStages - 2;
            const int stx = (st >= 2) ? st - 2 : st + kStages - 2;
            const uint32_t phx = ph ^ ((st >= 2) ? 1u : 0u) ^ 1u;
            if (!failed && nx < ntile_t) {
                if (nx >= kStages && !mbar_wait_bounded(&empty[stx], phx, kWaitLimitNs)) {
                    failed = true;
                } else {
                    issue(nx, stx);
                    my_issued = nx + 1;
                    if (lane == 0)
                        *s_issued = static_cast<int>(nx + 1);
                }
            }
        }
        if (!failed && !(mbar_wait_bounded(&ready[st], ph, kWaitLimitNs) &&
                         mbar_wait_bounded(&full[st], ph, kWaitLimitNs)))
            failed = true;
        if (failed) {
            atomicOr(p.status, kStatusTimeout);
            *s_abort = 1;
            break;
        }

        if (active) {
            const io_t* su = reinterpret_cast<const io_t*>(smem + Lay::OFF_U + st * Lay::ROWS);
            const dl_t* sdl = reinterpret_cast<const dl_t*>(smem + Lay::OFF_DL + st * Lay::ROWS_DL);
            const io_t* sz = reinterpret_cast<const io_t*>(smem + Lay::OFF_Z + st * Lay::ROWS);
            const int32_t* orow = reinterpret_cast<const int32_t*>(smem + Lay::OFF_OUT + st * Lay::OUT_STRIDE);
            float* yp_out = p.ypart ? p.ypart + out_base + tid : nullptr;
            io_t* o_out = static_cast<io_t*>(p.out) + out_base + tid;
            const st_t* bf = reinterpret_cast<const st_t*>(smem + Lay::OFF_BF + st * Lay::BF_STRIDE);
            const float4* B4 = reinterpret_cast<const float4*>(bf);
            const float4* C4 = reinterpret_cast<const float4*>(bf + kTile * NS);
            if (precise) {
                // h = (1 + expm1(Delta*A)) h + Bbar*u*B without rounding Abar to fp32, so the
                // per-step error does not grow with the memory length 1/|Delta*A|; Bbar is Delta,
                // or expm1(Delta*A)/A with the exact ZOH
                for (int r = 0; r < rows; ++r) {
                    const float uv =
                        conv_step(Io<io_t>::ld(su + (r ^ xmask) * DC + tid), std::true_type{});
                    const float dr = Io<dl_t>::ld(sdl + r * DC + tid);
                    const float x = DQ ? fmaf(dr, dscale, bias_raw) : dr + bias_raw;
                    const float spv = fmaxf(x, 0.f) + log1p_unit(ex2(-fabsf(x) * kLog2e));
                    const float dt = softplus ? spv : x;
                    const float w = dt * uv;
                    if constexpr (WIDE) {
                        // fp64 state and readout; the per-step factors stay fp32
                        const double wd = static_cast<double>(dt) * static_cast<double>(uv);
                        if (PHASE1)
                            dsum += static_cast<double>(dt);
                        double ypd = 0.0;
#pragma unroll
                        for (int n = 0; n < NS; ++n) {
                            const float em1 = expm1_acc(dt * a_l[n]);
                            const double wb = p.zoh && a_l[n] != 0.f
                                                  ? static_cast<double>(em1 / a_l[n]) * static_cast<double>(uv)
                                                  : wd;
                            const double hb = fma(wb, bf[r * NS + n], kst[n]);
                            kst[n] = fma(static_cast<double>(em1), kst[n], hb);
                            if (!PHASE1)
                                ypd = fma(bf[kTile * NS + r * NS + n], kst[n], ypd);
                        }
                        if (!PHASE1) {
                            float y = static_cast<float>(fma(static_cast<double>(dskip), static_cast<double>(uv), ypd));
                            if (YPART) {
                                yp_out[orow[r]] = y;
                            } else {
                                if (GATE) {
                                    const float zv = Io<io_t>::ld(sz + (r ^ xmask) * DC + tid);
                                    y *= zv / (1.f + ex2(-zv * kLog2e));
                                }
                                o_out[orow[r]] = Io<io_t>::st(y);
                            }
                        }
                        continue;
                    }
                    if (PHASE1)
                        dsum += dt * kLog2e;
                    float yp = 0.f;
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
                            const int n = n4 * 4 + j;
                            const float em1 = expm1_acc(dt * a_l[n]);
                            const float wb = p.zoh && a_l[n] != 0.f ? (em1 / a_l[n]) * uv : w;
                            kst[n] = fmaf(em1, kst[n], fmaf(wb, bv[j], kst[n]));
                            if (!PHASE1)
                                yp = fmaf(cv[j], kst[n], yp);
                        }
                    }
                    if (!PHASE1) {
                        float y = fmaf(dskip, uv, yp);
                        if (YPART) {
                            yp_out[orow[r]] = y;
                        } else {
                            if (GATE) {
                                const float zv = Io<io_t>::ld(sz + (r ^ xmask) * DC + tid);
                                y *= zv / (1.f + ex2(-zv * kLog2e));
                            }
                            o_out[orow[r]] = Io<io_t>::st(y);
                        }
                    }
                }
            } else if constexpr (!WIDE) {
                // fast path, kGroup rows at a time: first the per-step scalars of all kGroup
                // rows, then their state updates; no branch inside a group, so the compiler can
                // overlap consecutive rows.  A row past the tile's end leaves the state as it
                // is: q = 1, w = the previous w (so w_prev/w = 1), and B = 0 there.
                auto group = [&](auto chain_tag, auto full_tag, auto dirc_tag, int r0) {
                    constexpr bool CHAIN = decltype(chain_tag)::value;
                    constexpr bool FULL = decltype(full_tag)::value;  // all kGroup rows valid
                    // u/z row order inside the group: +1 ascending, -1 descending (the rows of
                    // an aligned group run linearly for every xmask), 0 = through xmask
                    constexpr int DIRC = decltype(dirc_tag)::value;
                    const int rowbase = r0 ^ xmask;  // u/z row of g = 0 when DIRC != 0
                    float s_q[kGroup], s_w[kGroup], s_rr[kGroup], s_sp[kGroup], s_du[kGroup],
                        s_g[kGroup];
#pragma unroll
                    for (int g = 0; g < kGroup; ++g) {
                        const bool valid = FULL || r0 + g < rows;
                        const int r = valid ? (r0 + g) : (rows - 1);
                        // (a row past the end shifts the convolution window, but it only occurs
                        // in the segment's last tile)
                        const int ur = DIRC == 0 ? (r ^ xmask) : rowbase + DIRC * g;
                        const float uv =
                            conv_step(Io<io_t>::ld(su + ur * DC + tid), std::false_type{});
                        const float dr = Io<dl_t>::ld(sdl + r * DC + tid);
                        // x = (delta + bias) * log2(e); Delta*log2(e) = softplus in base 2 of x
                        const float x = fmaf(dr, DQ ? dscale2 : kLog2e, bias2);
                        const float e = ex2(-fabsf(x));              // 2^-|x| in (0, 1]
                        const float l_big = lg2(1.f + e);
                        // log2(1+e) for small e: e*log2(e)*(1 - e/2), rel. error < e^2/3
                        const float l_small = e * fmaf(e, -0.5f * kLog2e, kLog2e);
                        const float spv = fmaxf(x, 0.f) + (e < 0.00390625f ? l_small : l_big);
                        const float sp2 = valid ? (softplus ? spv : x) : 0.f;
                        float w = sp2 * uv;                           // = Delta*u / ln 2
                        w = fabsf(w) < kTinyW ? kTinyW : w;
                        s_w[g] = valid ? w : (g == 0 ? wprev : s_w[g - 1]);
                        s_sp[g] = sp2;
                        s_q[g] = CHAIN ? ex2(sp2 * a_l[0]) : 1.f;
                        s_du[g] = dskip * uv;
                        s_g[g] = 1.f;
                        if (GATE) {
                            // silu(z) = z * sigmoid(z) = h + h * tanh(h) with h = z/2
                            const float hz = 0.5f * Io<io_t>::ld(sz + ur * DC + tid);
                            s_g[g] = fmaf(hz, tanh_approx(hz), hz);
                        }
                    }
#pragma unroll
                    for (int g = 0; g < kGroup; ++g)
                        s_rr[g] = (g == 0 ? wprev : s_w[g - 1]) * rcp(s_w[g]);
                    wprev = s_w[kGroup - 1];
#pragma unroll
                    for (int g = 0; g < kGroup; ++g) {
                        const int r = r0 + g;  // < kTile; rows past the tile end read B = C = 0
                        const float rr = s_rr[g];
                        if (PHASE1)
                            dsum += s_sp[g];
                        // c[n] = (w_prev/w) * exp(Delta*A[d,n]) as pairs (n, n+1)
                        float2 cp[NS / 2];
                        if (CHAIN) {
                            // q^(n+1): pair j = pair (j-1) * (q^2, q^2); the rows of a group are
                            // independent, so the chain's depth costs no issue slots
                            const float q = s_q[g];
                            const float q2 = q * q;
                            cp[0] = make_float2(rr * q, rr * q2);
                            const float2 qq = make_float2(q2, q2);
#pragma unroll
                            for (int j = 1; j < NS / 2; ++j)
                                cp[j] = __fmul2_rn(cp[j - 1], qq);
                        } else {
                            const float sp2 = s_sp[g];
#pragma unroll
                            for (int j = 0; j < NS / 2; ++j)
                                cp[j] = make_float2(rr * ex2(sp2 * a_l[2 * j]),
                                                    rr * ex2(sp2 * a_l[2 * j + 1]));
                        }
                        // C . k in two packed accumulators (fewer adds at the end than four),
                        // started by the products of the first four states (no zeroing)
                        float2 yacc[2];
#pragma unroll
                        for (int n4 = 0; n4 < NS / 4; ++n4) {
                            const float4 bq = B4[r * (NS / 4) + n4];
                            kst2[2 * n4] =
                                __ffma2_rn(cp[2 * n4], kst2[2 * n4], make_float2(bq.x, bq.y));
                            kst2[2 * n4 + 1] = __ffma2_rn(cp[2 * n4 + 1], kst2[2 * n4 + 1],
                                                          make_float2(bq.z, bq.w));
                            if (!PHASE1) {
                                const float4 cq = C4[r * (NS / 4) + n4];
                                if (n4 == 0) {
                                    yacc[0] = __fmul2_rn(make_float2(cq.x, cq.y), kst2[0]);
                                    yacc[1] = __fmul2_rn(make_float2(cq.z, cq.w), kst2[1]);
                                } else {
                                    yacc[0] = __ffma2_rn(make_float2(cq.x, cq.y),
                                                         kst2[2 * n4], yacc[0]);
                                    yacc[1] = __ffma2_rn(make_float2(cq.z, cq.w),
                                                         kst2[2 * n4 + 1], yacc[1]);
                                }
                            }
                        }
                        if (!PHASE1) {
                            const float2 ys = __fadd2_rn(yacc[0], yacc[1]);
                            float y = fmaf(s_w[g], ys.x + ys.y, s_du[g]);
                            if (FULL || r < rows) {
                                if (YPART) {
                                    yp_out[orow[r]] = y;
                                } else {
                                    if (GATE)
                                        y *= s_g[g];
                                    o_out[orow[r]] = Io<io_t>::st(y);
                                }
                            }
                        }
                    }
                };
                using Up = std::integral_constant<int, 1>;
                using Down = std::integral_constant<int, -1>;
                using Any = std::integral_constant<int, 0>;
                for (int r0 = 0; r0 < rows; r0 += kGroup) {
                    const bool full_group = r0 + kGroup <= rows;  // the same for the whole CTA
                    if (use_chain) {
                        // full groups with a fixed row order: row offsets become constants.  The
                        // multi-direction kernels run both orders at once and keep one copy of
                        // the code (two hot copies measured slower there).
                        if (full_group && !YPART) {
                            if (xmask == 0)
                                group(std::true_type{}, std::true_type{}, Up{}, r0);
                            else
                                group(std::true_type{}, std::true_type{}, Down{}, r0);
                        } else if (full_group) {
                            group(std::true_type{}, std::true_type{}, Any{}, r0);
                        } else {
                            group(std::true_type{}, std::false_type{}, Any{}, r0);
                        }
                    } else {
                        group(std::false_type{}, std::false_type{}, Any{}, r0);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[st]);
    }

    if (failed) {
        atomicOr(p.status, kStatusTimeout);
        *s_abort = 1;
        // let the copies this warp issued land before the CTA's shared memory goes away; the
        // waits are bounded as well
        if (lane == 0) {
            for (int64_t j = 0; j < my_issued; ++j) {
                const int issuer = j < kStages - 2 ? 0 : static_cast<int>((j - (kStages - 2)) % WARPS);
                if (issuer == warp)
                    (void)mbar_wait_bounded(&full[j % kStages],
                                            static_cast<uint32_t>((j / kStages) & 1), kWaitLimitNs / 8);
            }
        }
        return;
    }

    if (!active)
        return;
    if (PHASE1) {
        const int64_t ci = (kb * p.S + seg) * p.D + d;
        carry_s[ci] = dsum;
#pragma unroll
        for (int n = 0; n < NS; ++n)
            if (n < p.N)
                carry_h[ci * p.N + n] = static_cast<st_t>(wprev) * kst[n];
    } else if (p.last_state && seg == p.S - 1) {
        float* ls = p.last_state + (kb * p.D + d) * p.N;
#pragma unroll
        for (int n = 0; n < NS; ++n)
            if (n < p.N)
                ls[n] = static_cast<float>(static_cast<st_t>(wprev) * kst[n]);
    }
}

// ---------------------------------------------------------------------------- merge kernel

// Four adjacent channels per thread: 16-byte fp32 loads from every direction's plane, all issued
// before the sum; the partial outputs are read once, so loads and stores stream past L1/L2.
template <typename io_t> struct Io4;
template <> struct Io4<float> {
    static __device__ __forceinline__ float4 ld(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
    static __device__ __forceinline__ void st(float* p, float4 v) { __stcs(reinterpret_cast<float4*>(p), v); }
};
template <> struct Io4<__nv_bfloat16> {
    static __device__ __forceinline__ float4 ld(const __nv_bfloat16* p)
    {
        const uint2 w = __ldcs(reinterpret_cast<const uint2*>(p));
        return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                           __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
    }
    static __device__ __forceinline__ void st(__nv_bfloat16* p, float4 v)
    {
        const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
        const __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
        uint2 w;
        w.x = *reinterpret_cast<const uint32_t*>(&a);
        w.y = *reinterpret_cast<const uint32_t*>(&b);
        __stcs(reinterpret_cast<uint2*>(p), w);
    }
};

__device__ __forceinline__ float silu_f(float z) { return z * rcp(1.f + ex2(-z * kLog2e)); }

template <typename io_t, bool GATE, int K>
__global__ void __launch_bounds__(256) merge_kernel(const __grid_constant__ MergeParams p)
{
    pdl_wait();  // the per-direction outputs come from the scan launch just before
    const int64_t plane = p.rows * p.D;
    const int64_t n4 = plane / 4;  // D is a multiple of 4
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n4;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float4 part[K];
#pragma unroll
        for (int k = 0; k < K; ++k)
            part[k] = Io4<float>::ld(p.ypart + k * plane + 4 * i);
        float4 y = part[0];
#pragma unroll
        for (int k = 1; k < K; ++k) {
            y.x += part[k].x;
            y.y += part[k].y;
            y.z += part[k].z;
            y.w += part[k].w;
        }
        if (GATE) {
            const float4 zv = Io4<io_t>::ld(static_cast<const io_t*>(p.z) + 4 * i);
            y.x *= silu_f(zv.x);
            y.y *= silu_f(zv.y);
            y.z *= silu_f(zv.z);
            y.w *= silu_f(zv.w);
        }
        Io4<io_t>::st(static_cast<io_t*>(p.out) + 4 * i, y);
    }
}

// ---------------------------------------------------------------------------- dispatch

constexpr int kWarps = 2;

template <typename io_t, typename dl_t, int NS, bool GATE, bool PHASE1, bool YPART, bool CONV>
cudaError_t launch_t(const ScanParams& p, cudaStream_t stream, bool prepare_only)
{
    using Lay = Layout<io_t, dl_t, NS, kWarps, GATE, PHASE1, YPART ? 5 : 4>;
    auto kern = scan_kernel<io_t, dl_t, NS, kWarps, GATE, PHASE1, YPART, CONV>;
    if (prepare_only)
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::BYTES);
    const int64_t ntiles = (p.D + Lay::DC - 1) / Lay::DC;
    const int64_t nseg = PHASE1 ? (p.S - 1) : p.S;
    const int64_t nblocks = ntiles * nseg * p.batch * p.K;
    if (nblocks <= 0)
        return cudaSuccess;
    // a scan launch that follows the aggregate launch may start before it ends (its segment-0
    // CTAs need nothing from it; the others wait for it in the kernel)
    const bool after_aggregates = !PHASE1 && p.S > 1;
    return launch_ex(kern, static_cast<unsigned>(nblocks), 32 * kWarps, Lay::BYTES, stream,
                     after_aggregates, p);
}

template <typename io_t, typename dl_t, int NS, bool CONV>
cudaError_t launch_nc(const ScanParams& p, int phase1, cudaStream_t stream, bool prepare_only)
{
    if (phase1)
        return launch_t<io_t, dl_t, NS, false, true, false, CONV>(p, stream, prepare_only);
    if (p.ypart)
        return launch_t<io_t, dl_t, NS, false, false, true, CONV>(p, stream, prepare_only);
    return p.z ? launch_t<io_t, dl_t, NS, true, false, false, CONV>(p, stream, prepare_only)
               : launch_t<io_t, dl_t, NS, false, false, false, CONV>(p, stream, prepare_only);
}

template <typename io_t, typename dl_t, int NS>
cudaError_t launch_ns(const ScanParams& p, int phase1, cudaStream_t stream, bool prepare_only)
{
    return p.conv_w ? launch_nc<io_t, dl_t, NS, true>(p, phase1, stream, prepare_only)
                    : launch_nc<io_t, dl_t, NS, false>(p, phase1, stream, prepare_only);
}

// All scan launches of io type io_t with delta stored as dl_t (io_t, or int8_t codes); with
// prepare_only, only the kernel's shared-memory attribute is set (nothing is launched).
template <typename io_t, typename dl_t = io_t>
cudaError_t launch_io(const ScanParams& p, int phase1, cudaStream_t stream, bool prepare_only)
{
    if (p.N <= 4)
        return launch_ns<io_t, dl_t, 4>(p, phase1, stream, prepare_only);
    if (p.N <= 8)
        return launch_ns<io_t, dl_t, 8>(p, phase1, stream, prepare_only);
    return launch_ns<io_t, dl_t, 16>(p, phase1, stream, prepare_only);
}

}  // namespace

}  // namespace ss
