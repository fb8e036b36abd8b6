// The bfloat16 selective-scan kernel (S6 forward) for sm_100a: the hot path of the library.
//
// Work split.  One warp is one CTA and owns 64 adjacent channels of one (segment, direction,
// batch row); each lane keeps two adjacent channels, d and d+1, with their 16-state vectors in
// registers for the whole segment ("Understanding Mamba from zero" sec. 5: per channel and state
// the recurrence is a scalar affine map).  Two channels per lane let the per-step scalars
// (softplus, exp, the gate) run as packed f32x2 operations and make every broadcast load of a
// B or C tile serve both channels.
//
// Data movement.  The warp streams its inputs through a ring of kStages shared-memory stages of
// kTile = 16 steps.  Each stage is filled by asynchronous copies that complete on one mbarrier:
// a tensor-map box (cp.async.bulk.tensor) per tile for u, delta and z (the rows picked through
// the direction's index map: a 2D box for the row orders, 3D boxes of 8 image rows for the
// column orders, one bulk copy per row otherwise) and one bulk copy each for the B and C rows.
// At the start of tile i the warp converts that tile's B and C to fp32 once (into one buffer
// shared by the whole tile) and refills the stage of tile i-1 with tile i+kStages-1.  No other
// warp is involved: the lane that issues the copies is the only producer and the warp the only
// consumer.  With kTmaStore and a row order, a full tile's outputs go back through shared memory
// (into the rows of u the tile has consumed) and out with one tensor-map store per tile.
//
// Arithmetic (per step, fp32 state):
//   x = (delta + bias) * log2(e); Delta*log2(e) = softplus in base 2 of x
//   w = Delta*u*log2(e), clamped to |w| >= 2^-64 (see below); q = exp(Delta*A[d,0])
//   normalised state k = h / w:  k_n <- (w_prev / w) * Abar_n * k_n + ln2 * B_n
//   y = w * (C . k) + Dskip*u, then the silu(z) gate
// Abar_n = exp(Delta*A[d,n]) comes from the power chain q^(n+1) when A[d,n] = (n+1)*A[d,0]
// (checked per channel; warp-uniform), else from one ex2 per state.  This is three FP32
// operations per state update (chain multiply, state multiply-add, readout multiply-add), as
// packed f32x2 instructions over the state pairs.  A step whose |Delta*u| is below 2^-64
// (padding with u = 0, or Delta = 0) is normalised by 2^-64 instead, which adds at most
// 2^-64*|B_n| to that step's h_n; the state and outputs are otherwise exact up to rounding.
//
// Scheduling.  A full tile runs as groups of kGroup steps: the per-step scalars of group g+1
// (loads, softplus, exp, reciprocal, gate: MUFU- and ALU-heavy) are computed in the same
// straight-line block as the state updates of group g (FMA-heavy), so the two overlap.  A tile
// shorter than 16 steps (a sequence's end) and the generic-A form take a plain step-by-step
// path.
//
// Segments (the chunked scan of "S4 -> Mamba" sec. 2.2): the aggregate launch (MAIN = false)
// scans segments 0..S-2 from zero and stores each end state h and sum(Delta*log2 e); the main
// launch folds the carries of the segments before its own: h <- exp(A * sum Delta) * h + h_s.
//
// Every wait is bounded (2 s).  A wait that gives up sets the library's device error word, waits
// (bounded) for the copies still in flight, and the CTA returns.
#pragma once

#include <type_traits>

#include "ss_device.cuh"

namespace ss {

namespace {

namespace fast {
constexpr int kRows = kTile;      // steps per tile (16)
constexpr int kStages = 3;        // tiles in the ring
constexpr int kCh = 64;           // channels per CTA: one warp, two adjacent channels per lane
constexpr int kN = 16;            // state slots; a smaller N leaves the missing B and C at zero
constexpr int kGroup = 4;         // steps whose scalars are computed together
constexpr int kMinBlocks = 8;     // CTAs per SM the register budget is sized for
constexpr bool kTmaStore = false; // row orders: full tiles' outputs leave through a tensor store
}  // namespace fast

// cp.async.bulk.tensor store of a 2D box from shared memory, and the waits for bulk stores.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int32_t c0,
                                             int32_t c1)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_read_all()
{
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_all()
{
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

template <typename dl_t, bool MAIN, bool GATE, bool YPART>
struct FastLayout {
    static constexpr bool HAS_Z = MAIN && GATE && !YPART;
    static constexpr bool HAS_C = MAIN;
    static constexpr int U_BYTES = fast::kRows * fast::kCh * 2;
    static constexpr int DL_BYTES = fast::kRows * fast::kCh * static_cast<int>(sizeof(dl_t));
    // B/C rows are copied from a 16-byte aligned superset of the tile's rows
    static constexpr int BC_RAW = ((fast::kRows * fast::kN * 2 + 32 + 15) / 16) * 16;
    // one stage: u, delta, z tiles (tensor-copy destinations, 128-byte aligned), raw B and C
    static constexpr int S_U = 0;
    static constexpr int S_DL = S_U + U_BYTES;
    static constexpr int S_Z = S_DL + DL_BYTES;
    static constexpr int S_BR = S_Z + (HAS_Z ? U_BYTES : 0);
    static constexpr int S_CR = S_BR + BC_RAW;
    static constexpr int STAGE = ((S_CR + (HAS_C ? BC_RAW : 0) + 127) / 128) * 128;
    // per CTA: the current tile's fp32 B and C, its output row offsets, the barriers
    static constexpr int OFF_BF = fast::kStages * STAGE;
    static constexpr int OFF_CF = OFF_BF + fast::kRows * fast::kN * 4;
    static constexpr int OFF_OROW = OFF_CF + (HAS_C ? fast::kRows * fast::kN * 4 : 0);
    static constexpr int OFF_BAR = OFF_OROW + fast::kRows * 4;
    static constexpr int BYTES = OFF_BAR + fast::kStages * 8;
    static_assert(U_BYTES % 128 == 0 && DL_BYTES % 128 == 0 && S_BR % 16 == 0 && S_CR % 16 == 0 &&
                      OFF_BF % 16 == 0 && OFF_BAR % 8 == 0,
                  "copy destinations need 128-byte (tensor) / 16-byte (bulk) alignment");
};

// bf16 pair (low half = first element) as two floats
__device__ __forceinline__ float2 bf2_unpack(uint32_t w)
{
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Two int8 codes (bits 0-7 and 8-15) as exact floats: offset-binary code + 2^23 placed in the
// mantissa of 2^23, then 2^23 + 128 subtracted (exact).
__device__ __forceinline__ float2 i8x2_unpack(uint32_t v)
{
    const uint32_t x = v ^ 0x8080u;
    const float a = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7540));
    const float b = __uint_as_float(__byte_perm(x, 0x4B000000u, 0x7541));
    return __fadd2_rn(make_float2(a, b), make_float2(-8388736.f, -8388736.f));
}

__device__ __forceinline__ uint32_t bf2_pack(float2 y)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(y.x, y.y);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// Per-step values of one step for the lane's two channels.
struct RowScal {
    float2 rr;  // w_prev / w
    float2 q;   // exp(Delta * A[d,0])
    float2 wg;  // w * gate (readout scale)
    float2 dg;  // Dskip * u * gate
};

template <typename dl_t, bool MAIN, bool GATE, bool YPART, bool CONV>
__global__ void __launch_bounds__(32, fast::kMinBlocks)
    fast_scan_kernel(const __grid_constant__ ScanParams p)
{
    using Lay = FastLayout<dl_t, MAIN, GATE, YPART>;
    constexpr bool DQ = std::is_same<dl_t, int8_t>::value;  // int8 delta codes
    constexpr bool HAS_Z = Lay::HAS_Z;
    constexpr int ROWS = fast::kRows;
    constexpr int NSTG = fast::kStages;
    constexpr int CH = fast::kCh;
    constexpr int NS = fast::kN;
    constexpr int G = fast::kGroup;
    constexpr int NG = ROWS / G;
    constexpr bool TSTORE = fast::kTmaStore && MAIN && !YPART;
    static_assert(ROWS % G == 0 && NG % 2 == 0, "groups alternate between two register sets");

    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
    float* s_bf = reinterpret_cast<float*>(smem + Lay::OFF_BF);
    float* s_cf = reinterpret_cast<float*>(smem + Lay::OFF_CF);
    int32_t* s_orow = reinterpret_cast<int32_t*>(smem + Lay::OFF_OROW);
    const int lane = threadIdx.x;

    // ---- the CTA's (segment, direction, batch row, channel tile); segments are the slowest
    // index, so a main launch's segment-0 CTAs (which need no carry) come first
    const int64_t ntiles = (p.D + CH - 1) / CH;
    const int64_t per_seg = ntiles * p.batch * p.K;
    int64_t blk = blockIdx.x;
    const int seg = static_cast<int>(blk / per_seg);
    blk -= static_cast<int64_t>(seg) * per_seg;
    const int64_t tile = blk % ntiles;
    blk /= ntiles;
    const int64_t b = blk % p.batch;
    const int k = static_cast<int>(blk / p.batch);
    const int dir = k == 0 ? p.dirs[0] : k == 1 ? p.dirs[1] : k == 2 ? p.dirs[2] : p.dirs[3];
    const int64_t d0 = tile * CH;
    const int64_t dA = d0 + 2 * lane;  // this lane's channels dA and dA + 1
    const bool active = dA < p.D;      // D is even: both channels or neither
    const int dcv = static_cast<int>((p.D - d0) < CH ? (p.D - d0) : CH);
    const int64_t t_begin = static_cast<int64_t>(seg) * p.seg_len;
    const int64_t t_end = (t_begin + p.seg_len < p.L) ? (t_begin + p.seg_len) : p.L;
    const int64_t ntile_t = (t_end - t_begin + ROWS - 1) / ROWS;
    const int64_t kb = static_cast<int64_t>(k) * p.batch + b;  // (direction, batch) row block
    const int64_t ub = p.u_per_dir ? kb : b;                   // row block of this CTA's u
    const int64_t N = p.N;

    if (lane == 0) {
        for (int s = 0; s < NSTG; ++s)
            mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncwarp();
    // the next launch (the main scan after the aggregates, the merge after the scan) may start;
    // it waits for this grid's results itself where it needs them
    pdl_launch_dependents();
    if (p.test_timeout) {
        // failure-detection test hook: nothing completes full[0], so this bounded wait gives
        // up; no copy has been issued, so the CTA returns at once
        if (!mbar_wait_bounded(&full[0], 0, kTestWaitNs) && lane == 0)
            atomicOr(p.status, kStatusTimeout);
        return;
    }

    const __nv_bfloat16* gu = static_cast<const __nv_bfloat16*>(p.u);
    const __nv_bfloat16* gB = static_cast<const __nv_bfloat16*>(p.B);
    const __nv_bfloat16* gC = static_cast<const __nv_bfloat16*>(p.C);

    // ---- copies of one tile
    const int umode = (dir == SS_DIR_FWD || dir == SS_DIR_REV) ? 0 : (p.col3d ? 1 : 2);
    // step t0 + r of a tile reads u/z row (r ^ xmask) of its stage; delta rows are in scan order
    const int xmask = dir == SS_DIR_REV ? (ROWS - 1) : (dir == SS_DIR_COL_REV && umode == 1 ? 7 : 0);
    const uint32_t row_bytes = static_cast<uint32_t>(dcv) * 2u;
    constexpr uint32_t kBox2 = CH * ROWS * 2;
    constexpr uint32_t kBoxDL = CH * ROWS * sizeof(dl_t);
    constexpr uint32_t kBox3 = CH * 8 * 2;
    constexpr uint32_t kUZ = HAS_Z ? 2u : 1u;
    // first spatial row of the u/z box of the tile starting at step t0 (row orders)
    auto box_row = [&](int64_t t0) { return dir == SS_DIR_FWD ? t0 : p.L - t0 - ROWS; };

    auto bc_src = [&](const __nv_bfloat16* base, int64_t t0, int rows, uint32_t& bytes, int& skip) {
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(base + (kb * p.L + t0) * N);
        const uintptr_t a1 = reinterpret_cast<uintptr_t>(base + (kb * p.L + t0 + rows) * N);
        const uintptr_t lo = a0 & ~static_cast<uintptr_t>(15);
        const uintptr_t hi = (a1 + 15) & ~static_cast<uintptr_t>(15);
        bytes = static_cast<uint32_t>(hi - lo);
        skip = static_cast<int>((a0 - lo) / 2);
        return reinterpret_cast<const void*>(lo);
    };
    auto tile_rows = [&](int64_t it) {
        const int64_t t0 = t_begin + it * ROWS;
        return static_cast<int>((t_end - t0) < ROWS ? (t_end - t0) : ROWS);
    };

    // Fill the stage of tile `it` (all lanes call; lane 0 issues, plus per-row copies).
    auto issue = [&](int64_t it) {
        const int st = static_cast<int>(it % NSTG);
        unsigned char* sb = smem + st * Lay::STAGE;
        const int64_t t0 = t_begin + it * ROWS;
        const int rows = tile_rows(it);
        uint32_t bbytes, cbytes = 0;
        int bskip, cskip;
        const void* bsrc = bc_src(gB, t0, rows, bbytes, bskip);
        const void* csrc = Lay::HAS_C ? bc_src(gC, t0, rows, cbytes, cskip) : nullptr;
        if (lane == 0) {
            uint32_t tx = kBoxDL + bbytes + cbytes;
            if (umode == 0)
                tx += kUZ * kBox2;
            else if (umode == 1)
                tx += kUZ * kBox3 * static_cast<uint32_t>(rows / 8);
            else
                tx += kUZ * static_cast<uint32_t>(rows) * row_bytes;
            mbar_expect_tx(&full[st], tx);
            tma_2d(sb + Lay::S_DL, &p.tm_dl, static_cast<int32_t>(d0),
                   static_cast<int32_t>(kb * p.L + t0), &full[st]);
            if (umode == 0) {
                // reverse order: the box ends at the row of step t0
                const int64_t prow = box_row(t0);
                tma_2d(sb + Lay::S_U, &p.tm_u, static_cast<int32_t>(d0),
                       static_cast<int32_t>(ub * p.L + prow), &full[st]);
                if (HAS_Z)
                    tma_2d(sb + Lay::S_Z, &p.tm_z, static_cast<int32_t>(d0),
                           static_cast<int32_t>(b * p.L + prow), &full[st]);
            } else if (umode == 1) {
                for (int sub = 0; sub < rows / 8; ++sub) {
                    const int64_t tt = t0 + 8 * sub;
                    // column-major index of the lowest image row of the box
                    const int64_t c = dir == SS_DIR_COL ? tt : (p.L - 8 - tt);
                    const int64_t j = c / p.H, i = c - (c / p.H) * p.H;
                    tma_3d(sb + Lay::S_U + 8 * sub * CH * 2, &p.tm_u3, static_cast<int32_t>(d0),
                           static_cast<int32_t>(j), static_cast<int32_t>(ub * p.H + i), &full[st]);
                    if (HAS_Z)
                        tma_3d(sb + Lay::S_Z + 8 * sub * CH * 2, &p.tm_z3, static_cast<int32_t>(d0),
                               static_cast<int32_t>(j), static_cast<int32_t>(b * p.H + i), &full[st]);
                }
            }
            bulk_g2s(sb + Lay::S_BR, bsrc, bbytes, &full[st]);
            if (Lay::HAS_C)
                bulk_g2s(sb + Lay::S_CR, csrc, cbytes, &full[st]);
        }
        if (umode == 2) {
            __syncwarp();  // the transaction count is expected before any row copy completes
            for (int r = lane; r < rows; r += 32) {
                const int64_t pp = position(dir, p.L, p.H, p.W, t0 + r);
                bulk_g2s(sb + Lay::S_U + r * CH * 2, gu + (ub * p.L + pp) * p.D + d0, row_bytes,
                         &full[st]);
                if (HAS_Z)
                    bulk_g2s(sb + Lay::S_Z + r * CH * 2,
                             static_cast<const __nv_bfloat16*>(p.z) + (b * p.L + pp) * p.D + d0,
                             row_bytes, &full[st]);
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&full[st]);
    };

    // Tile `it`'s B (and C) as fp32 in the CTA's buffers, B carrying the ln 2 of the
    // normalised state; rows past the tile's end and states past N are zero.  With MAIN, also
    // the tile's output row offsets (in pairs of elements).
    auto convert = [&](int64_t it) {
        const int st = static_cast<int>(it % NSTG);
        const unsigned char* sb = smem + st * Lay::STAGE;
        const int64_t t0 = t_begin + it * ROWS;
        const int rows = tile_rows(it);
        uint32_t bytes;
        int bskip = 0, cskip = 0;
        bc_src(gB, t0, rows, bytes, bskip);
        if (Lay::HAS_C)
            bc_src(gC, t0, rows, bytes, cskip);
        const __nv_bfloat16* br = reinterpret_cast<const __nv_bfloat16*>(sb + Lay::S_BR) + bskip;
        const __nv_bfloat16* cr = reinterpret_cast<const __nv_bfloat16*>(sb + Lay::S_CR) + cskip;
        if (N == NS && bskip == 0 && cskip == 0) {
            // 16 rows of 16 values per tensor: lane l converts 8 values (16 bytes) of each
            static_assert(ROWS * NS * 2 == 32 * 16, "one 16-byte chunk per lane and tensor");
            const bool ok = (lane >> 1) < rows;
            auto cvt8 = [&](const __nv_bfloat16* src, float* dst, float scale) {
                const uint4 w = *reinterpret_cast<const uint4*>(src + 8 * lane);
                const float2 f0 = bf2_unpack(w.x), f1 = bf2_unpack(w.y), f2 = bf2_unpack(w.z),
                             f3 = bf2_unpack(w.w);
                float4* d4 = reinterpret_cast<float4*>(dst + 8 * lane);
                d4[0] = ok ? make_float4(f0.x * scale, f0.y * scale, f1.x * scale, f1.y * scale)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
                d4[1] = ok ? make_float4(f2.x * scale, f2.y * scale, f3.x * scale, f3.y * scale)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            };
            cvt8(br, s_bf, kLn2);
            if (Lay::HAS_C)
                cvt8(cr, s_cf, 1.f);
        } else {
            const unsigned short* brs = reinterpret_cast<const unsigned short*>(br);
            const unsigned short* crs = reinterpret_cast<const unsigned short*>(cr);
            for (int idx = lane; idx < ROWS * NS; idx += 32) {
                const int r = idx / NS, n = idx - (idx / NS) * NS;
                const bool ok = r < rows && n < N;
                s_bf[idx] = ok ? __uint_as_float(static_cast<uint32_t>(brs[r * N + n]) << 16) * kLn2
                               : 0.f;
                if (Lay::HAS_C)
                    s_cf[idx] = ok ? __uint_as_float(static_cast<uint32_t>(crs[r * N + n]) << 16) : 0.f;
            }
        }
        if (MAIN && lane < ROWS)
            s_orow[lane] = lane < rows
                               ? static_cast<int32_t>(position(dir, p.L, p.H, p.W, t0 + lane) * (p.D / 2))
                               : 0;
    };

    // ---- per-channel constants, as pairs over the lane's two channels
    const int64_t pk = p.params_per_dir ? static_cast<int64_t>(k) : 0;
    const float* Ak = p.A + pk * p.D * N;  // [D, N] of this direction's parameter set
    float2 bias2 = make_float2(0.f, 0.f), a02 = make_float2(0.f, 0.f), dsk2 = make_float2(0.f, 0.f);
    float2 sc2 = make_float2(kLog2e, kLog2e);  // multiplies delta_raw (int8: scale * log2 e)
    bool chain = true;  // A[d, n] == (n+1) * A[d, 0] for both channels
    if (active) {
        float a0[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const float* ar = Ak + (dA + c) * N;
            a0[c] = ar[0];
            for (int n = 1; n < N; ++n)
                if (ar[n] != static_cast<float>(n + 1) * a0[c])
                    chain = false;
            // with fewer than NS states, a growing chain could overflow in the unused slots
            if (N < NS && a0[c] > 0.f)
                chain = false;
        }
        a02 = make_float2(a0[0], a0[1]);
        if (p.Dskip)
            dsk2 = make_float2(p.Dskip[pk * p.D + dA], p.Dskip[pk * p.D + dA + 1]);
        if (p.bias)
            bias2 = make_float2(p.bias[pk * p.D + dA] * kLog2e, p.bias[pk * p.D + dA + 1] * kLog2e);
        if (DQ)
            sc2 = make_float2(p.delta_scale[dA] * kLog2e, p.delta_scale[dA + 1] * kLog2e);
    }
    const bool use_chain = __all_sync(0xffffffffu, chain) && !p.force_generic;
    const bool softplus = p.softplus != 0;

    // ---- causal depthwise convolution along the direction's scan order (CONV): taps and bias
    // halved (exact) and right-aligned so that cw[3] multiplies the current step; the inputs of
    // the three steps before the segment (zero before step 0) come from global memory once
    float2 cw[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                    make_float2(0.f, 0.f)};
    float2 cbias = make_float2(0.f, 0.f);
    float2 xm1 = make_float2(0.f, 0.f), xm2 = xm1, xm3 = xm1;  // inputs of steps t-1, t-2, t-3
    if (CONV && active) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const float* wk = p.conv_w + (static_cast<int64_t>(k) * p.D + dA + c) * p.conv_width;
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const int j = s - (4 - p.conv_width);
                const float v = j >= 0 ? 0.5f * wk[j] : 0.f;
                if (c == 0)
                    cw[s].x = v;
                else
                    cw[s].y = v;
            }
            const float cb = p.conv_b ? 0.5f * p.conv_b[static_cast<int64_t>(k) * p.D + dA + c] : 0.f;
            if (c == 0)
                cbias.x = cb;
            else
                cbias.y = cb;
        }
        auto halo = [&](int64_t t) {
            if (t < 0)
                return make_float2(0.f, 0.f);
            const int64_t pp = position(dir, p.L, p.H, p.W, t);
            return bf2_unpack(*reinterpret_cast<const uint32_t*>(gu + (ub * p.L + pp) * p.D + dA));
        };
        xm1 = halo(t_begin - 1);
        xm2 = halo(t_begin - 2);
        xm3 = halo(t_begin - 3);
    }

    // ---- state: k = h / w_prev as pairs (n, n+1), starting with w_prev = 1 (k = h)
    float2 ks[2][NS / 2];
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int j = 0; j < NS / 2; ++j)
            ks[c][j] = make_float2(0.f, 0.f);
    float2 wprev = make_float2(1.f, 1.f);
    float2 dsum = make_float2(0.f, 0.f);  // sum of Delta*log2(e) over the segment (aggregates)
    auto set_state = [&](int c, int n, float v) {
#pragma unroll
        for (int j = 0; j < NS / 2; ++j) {
            if (n == 2 * j) {
                if (c == 0) ks[0][j].x = v; else ks[1][j].x = v;
            } else if (n == 2 * j + 1) {
                if (c == 0) ks[0][j].y = v; else ks[1][j].y = v;
            }
        }
    };
    auto get_state = [&](int c, int n) {
        float v = 0.f;
#pragma unroll
        for (int j = 0; j < NS / 2; ++j) {
            if (n == 2 * j)
                v = c == 0 ? ks[0][j].x : ks[1][j].x;
            else if (n == 2 * j + 1)
                v = c == 0 ? ks[0][j].y : ks[1][j].y;
        }
        return v;
    };
    if (MAIN && active && p.init_state) {
        const float* h0 = p.init_state + (kb * p.D + dA) * N;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int n = 0; n < NS; ++n)
                if (n < N)
                    set_state(c, n, h0[c * N + n]);
    }
    if (MAIN && seg > 0)
        pdl_wait();  // the carries come from the aggregate launch just before this one
    if (MAIN && seg > 0 && active) {
        // fold the carries of segments 0..seg-1: h <- exp(A * sumDelta_s) * h + h_s
        for (int s = 0; s < seg; ++s) {
            const int64_t ci = (kb * p.S + s) * p.D + dA;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const float sd = __ldcg(p.carry_s + ci + c);
                const float* ch = p.carry_h + (ci + c) * N;
                const float* ar = Ak + (dA + c) * N;
#pragma unroll
                for (int n = 0; n < NS; ++n)
                    if (n < N)
                        set_state(c, n, ex2(ar[n] * sd) * get_state(c, n) + __ldcg(ch + n));
            }
        }
    }

    // ---- one step's scalars (from the raw words of u, delta, z of the lane's two channels)
    auto scal = [&](uint32_t uw, uint32_t dw, uint32_t zw, RowScal& s, float2& sp_out) {
        float2 u = bf2_unpack(uw);
        if (CONV) {
            // u <- silu(conv) = c/2 + c/2 * tanh(c/2) with the halved taps giving c/2 directly
            const float2 h = __ffma2_rn(cw[3], u, __ffma2_rn(cw[2], xm1, __ffma2_rn(cw[1], xm2,
                                                             __ffma2_rn(cw[0], xm3, cbias))));
            xm3 = xm2;
            xm2 = xm1;
            xm1 = u;
            u = __ffma2_rn(h, make_float2(tanh_approx(h.x), tanh_approx(h.y)), h);
        }
        const float2 dr = DQ ? i8x2_unpack(dw) : bf2_unpack(dw);
        const float2 x = __ffma2_rn(dr, sc2, bias2);
        const float e0 = ex2(-fabsf(x.x)), e1 = ex2(-fabsf(x.y));  // 2^-|x| in (0, 1]
        const float2 e = make_float2(e0, e1);
        const float2 ope = __fadd2_rn(e, make_float2(1.f, 1.f));
        // log2(1 + e) for small e: e*log2(e)*(1 - e/2), relative error < e^2/3
        const float2 ls = __fmul2_rn(e, __ffma2_rn(e, make_float2(-0.5f * kLog2e, -0.5f * kLog2e),
                                                   make_float2(kLog2e, kLog2e)));
        const float l0 = e0 < 0.00390625f ? ls.x : lg2(ope.x);
        const float l1 = e1 < 0.00390625f ? ls.y : lg2(ope.y);
        float2 sp = __fadd2_rn(make_float2(fmaxf(x.x, 0.f), fmaxf(x.y, 0.f)), make_float2(l0, l1));
        if (!softplus)
            sp = x;
        sp_out = sp;
        float2 w = __fmul2_rn(sp, u);  // Delta * u * log2(e)
        w.x = fabsf(w.x) < kTinyW ? kTinyW : w.x;
        w.y = fabsf(w.y) < kTinyW ? kTinyW : w.y;
        const float2 qa = __fmul2_rn(sp, a02);
        s.q = make_float2(ex2(qa.x), ex2(qa.y));
        s.rr = __fmul2_rn(wprev, make_float2(rcp(w.x), rcp(w.y)));
        wprev = w;
        if (!MAIN) {
            dsum = __fadd2_rn(dsum, sp);
            return;
        }
        const float2 du = __fmul2_rn(dsk2, u);
        if (HAS_Z) {
            // silu(z) = z * sigmoid(z) = h + h * tanh(h) with h = z/2
            const float2 hz = __fmul2_rn(make_float2(0.5f, 0.5f), bf2_unpack(zw));
            const float2 g = __ffma2_rn(hz, make_float2(tanh_approx(hz.x), tanh_approx(hz.y)), hz);
            s.wg = __fmul2_rn(w, g);
            s.dg = __fmul2_rn(du, g);
        } else {
            s.wg = w;
            s.dg = du;
        }
    };

    float2* const yp2 = YPART ? reinterpret_cast<float2*>(p.ypart) + ((kb * p.L) * p.D + d0) / 2 + lane
                              : nullptr;
    uint32_t* const o2 = (MAIN && !YPART)
                             ? reinterpret_cast<uint32_t*>(p.out) + ((b * p.L) * p.D + d0) / 2 + lane
                             : nullptr;

    // Readout of step r of the current tile, y = w * (C . k) + Dskip*u gated, and its store:
    // into the consumed u row of the stage (su_out, for a tensor store of the tile) or straight
    // to global memory.
    auto finish = [&](const RowScal& s, const float2 ys, int r, uint32_t* su_out) {
        const float2 y = __ffma2_rn(s.wg, ys, s.dg);
        if (TSTORE && su_out) {
            su_out[(r ^ xmask) * (CH / 2)] = bf2_pack(y);
            return;
        }
        const int32_t off = s_orow[r];
        if (active) {
            if (YPART)
                yp2[off] = y;
            else
                o2[off] = bf2_pack(y);
        }
    };

    // State update (power chain) and readout of step r of the current tile.  State pairs outer,
    // channels inner: each B/C vector is live only while both channels use it.
    auto upd_chain = [&](const RowScal& s, int r, uint32_t* su_out) {
        const float4* B4 = reinterpret_cast<const float4*>(s_bf) + r * (NS / 4);
        const float4* C4 = reinterpret_cast<const float4*>(s_cf) + r * (NS / 4);
        // c_n = (w_prev/w) * q^(n+1) as pairs: pair j = pair (j-1) * (q^2, q^2)
        const float q2a = s.q.x * s.q.x, q2b = s.q.y * s.q.y;
        const float rqa = s.rr.x * s.q.x, rqb = s.rr.y * s.q.y;
        float2 Pa = make_float2(rqa, rqa * s.q.x), Pb = make_float2(rqb, rqb * s.q.y);
        const float2 QQa = make_float2(q2a, q2a), QQb = make_float2(q2b, q2b);
        float2 a0a = make_float2(0.f, 0.f), a1a = a0a, a0b = a0a, a1b = a0a;
#pragma unroll
        for (int i = 0; i < NS / 4; ++i) {
            const float4 bv = B4[i];
            float4 cv = make_float4(0.f, 0.f, 0.f, 0.f);
            if (MAIN)
                cv = C4[i];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = 2 * i + h;
                if (j > 0) {
                    Pa = __fmul2_rn(Pa, QQa);
                    Pb = __fmul2_rn(Pb, QQb);
                }
                const float2 bj = h ? make_float2(bv.z, bv.w) : make_float2(bv.x, bv.y);
                ks[0][j] = __ffma2_rn(Pa, ks[0][j], bj);
                ks[1][j] = __ffma2_rn(Pb, ks[1][j], bj);
                if (MAIN) {
                    const float2 cj = h ? make_float2(cv.z, cv.w) : make_float2(cv.x, cv.y);
                    if (j == 0) {
                        a0a = __fmul2_rn(cj, ks[0][j]);
                        a0b = __fmul2_rn(cj, ks[1][j]);
                    } else if (j == 1) {
                        a1a = __fmul2_rn(cj, ks[0][j]);
                        a1b = __fmul2_rn(cj, ks[1][j]);
                    } else if (h) {
                        a1a = __ffma2_rn(cj, ks[0][j], a1a);
                        a1b = __ffma2_rn(cj, ks[1][j], a1b);
                    } else {
                        a0a = __ffma2_rn(cj, ks[0][j], a0a);
                        a0b = __ffma2_rn(cj, ks[1][j], a0b);
                    }
                }
            }
        }
        if (MAIN) {
            const float2 sa = __fadd2_rn(a0a, a1a), sb = __fadd2_rn(a0b, a1b);
            finish(s, make_float2(sa.x + sa.y, sb.x + sb.y), r, su_out);
        }
    };

    // Generic A: Abar_n = exp(Delta*A[d,n]) with one ex2 per state, A read through L1 (a
    // fallback that keeps the register budget of the power-chain form).
    auto upd_generic = [&](const RowScal& s, const float2 sp, int r) {
        const float2* B2 = reinterpret_cast<const float2*>(s_bf) + r * (NS / 2);
        const float2* C2 = reinterpret_cast<const float2*>(s_cf) + r * (NS / 2);
        float2 ys = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const float rr = c == 0 ? s.rr.x : s.rr.y;
            const float spc = c == 0 ? sp.x : sp.y;
            const float* ac = Ak + (dA + c) * N;
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < NS / 2; ++j) {
                // states past N have B = C = 0 and A read as 0 (factor 1)
                const float e0 = active && 2 * j < N ? __ldg(ac + 2 * j) : 0.f;
                const float e1 = active && 2 * j + 1 < N ? __ldg(ac + 2 * j + 1) : 0.f;
                const float2 P = make_float2(rr * ex2(spc * e0), rr * ex2(spc * e1));
                ks[c][j] = __ffma2_rn(P, ks[c][j], B2[j]);
                if (MAIN)
                    acc = __ffma2_rn(C2[j], ks[c][j], acc);
            }
            if (c == 0)
                ys.x = acc.x + acc.y;
            else
                ys.y = acc.x + acc.y;
        }
        if (MAIN)
            finish(s, ys, r, nullptr);
    };

    // ---- the tiles
    bool failed = false;
    int64_t issued = 0;
    for (; issued < NSTG - 1 && issued < ntile_t; ++issued)
        issue(issued);
    int64_t it = 0;
    for (; it < ntile_t; ++it) {
        const int st = static_cast<int>(it % NSTG);
        if (!mbar_wait_bounded(&full[st], static_cast<uint32_t>((it / NSTG) & 1), kWaitLimitNs)) {
            failed = true;
            break;
        }
        convert(it);
        __syncwarp();
        // the stage of tile it-1 (finished by every lane) receives tile it+NSTG-1, once a
        // tensor store of tile it-1's outputs has read them from it
        if (issued < ntile_t && issued == it + NSTG - 1) {
            if (TSTORE && lane == 0)
                bulk_wait_read_all();
            issue(issued);
            ++issued;
        }
        unsigned char* sb = smem + st * Lay::STAGE;
        uint32_t* su = reinterpret_cast<uint32_t*>(sb + Lay::S_U) + lane;
        const uint32_t* sz = reinterpret_cast<const uint32_t*>(sb + Lay::S_Z) + lane;
        const uint32_t* sd32 = reinterpret_cast<const uint32_t*>(sb + Lay::S_DL) + lane;
        const unsigned short* sd16 = reinterpret_cast<const unsigned short*>(sb + Lay::S_DL) + lane;
        auto dword = [&](int r) -> uint32_t {
            return DQ ? static_cast<uint32_t>(sd16[r * (CH / 2)]) : sd32[r * (CH / 2)];
        };
        auto scal_row = [&](int r, RowScal& s, float2& sp) {
            const int ur = r ^ xmask;
            scal(su[ur * (CH / 2)], dword(r), HAS_Z ? sz[ur * (CH / 2)] : 0u, s, sp);
        };
        const int rows = tile_rows(it);
        if (rows == ROWS && use_chain) {
            // full tile: the scalars of group g+1 next to the updates of group g
            uint32_t* su_out = (TSTORE && umode == 0) ? su : nullptr;
            RowScal SA[G], SB[G];
            float2 spd;
#pragma unroll
            for (int g = 0; g < G; ++g)
                scal_row(g, SA[g], spd);
#pragma unroll
            for (int gi = 0; gi < NG; ++gi) {
                if (gi + 1 < NG) {
#pragma unroll
                    for (int g = 0; g < G; ++g)
                        scal_row((gi + 1) * G + g, (gi & 1) ? SA[g] : SB[g], spd);
                }
#pragma unroll
                for (int g = 0; g < G; ++g)
                    upd_chain((gi & 1) ? SB[g] : SA[g], gi * G + g, su_out);
            }
            if (TSTORE && umode == 0) {
                // the tile's outputs, now in its u rows, leave with one tensor store
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0)
                    tma_store_2d(&p.tm_out, sb + Lay::S_U, static_cast<int32_t>(d0),
                                 static_cast<int32_t>(b * p.L + box_row(t_begin + it * ROWS)));
            }
        } else if (use_chain) {
            for (int r = 0; r < rows; ++r) {
                RowScal s;
                float2 sp;
                scal_row(r, s, sp);
                upd_chain(s, r, nullptr);
            }
        } else {
            for (int r = 0; r < rows; ++r) {
                RowScal s;
                float2 sp;
                scal_row(r, s, sp);
                upd_generic(s, sp, r);
            }
        }
        // every lane is done with this tile's stage and fp32 B/C before they are reused
        fence_proxy_async_smem();
        __syncwarp();
    }
    if (TSTORE && lane == 0)
        bulk_wait_all();  // the tensor stores have completed before the CTA ends

    if (failed) {
        atomicOr(p.status, kStatusTimeout);
        // let the copies still in flight land before the CTA's shared memory goes away
        if (lane == 0)
            for (int64_t j = it; j < issued; ++j)
                (void)mbar_wait_bounded(&full[j % NSTG], static_cast<uint32_t>((j / NSTG) & 1),
                                        kWaitLimitNs / 8);
        return;
    }
    if (!active)
        return;
    if (!MAIN) {
        const int64_t ci = (kb * p.S + seg) * p.D + dA;
        p.carry_s[ci] = dsum.x;
        p.carry_s[ci + 1] = dsum.y;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const float wl = c == 0 ? wprev.x : wprev.y;
#pragma unroll
            for (int n = 0; n < NS; ++n)
                if (n < N)
                    p.carry_h[(ci + c) * N + n] = wl * get_state(c, n);
        }
    } else if (p.last_state && seg == p.S - 1) {
        float* ls = p.last_state + (kb * p.D + dA) * N;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const float wl = c == 0 ? wprev.x : wprev.y;
#pragma unroll
            for (int n = 0; n < NS; ++n)
                if (n < N)
                    ls[c * N + n] = wl * get_state(c, n);
        }
    }
}

// ---------------------------------------------------------------------------- launch

template <typename dl_t, bool MAIN, bool GATE, bool YPART, bool CONV>
cudaError_t fast_launch_t(const ScanParams& p, cudaStream_t stream, bool prepare_only)
{
    using Lay = FastLayout<dl_t, MAIN, GATE, YPART>;
    auto kern = fast_scan_kernel<dl_t, MAIN, GATE, YPART, CONV>;
    if (prepare_only)
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::BYTES);
    const int64_t ntiles = (p.D + fast::kCh - 1) / fast::kCh;
    const int64_t nseg = MAIN ? p.S : (p.S - 1);
    const int64_t nblocks = ntiles * nseg * p.batch * p.K;
    if (nblocks <= 0)
        return cudaSuccess;
    // a main launch that follows the aggregate launch may start before it ends (its segment-0
    // CTAs need nothing from it; the others wait for it in the kernel)
    return launch_ex(kern, static_cast<unsigned>(nblocks), 32, Lay::BYTES, stream,
                     MAIN && p.S > 1, p);
}

template <typename dl_t, bool CONV>
cudaError_t fast_launch_c(const ScanParams& p, int phase1, cudaStream_t stream, bool prepare_only)
{
    if (phase1)
        return fast_launch_t<dl_t, false, false, false, CONV>(p, stream, prepare_only);
    if (p.ypart)
        return fast_launch_t<dl_t, true, false, true, CONV>(p, stream, prepare_only);
    return p.z ? fast_launch_t<dl_t, true, true, false, CONV>(p, stream, prepare_only)
               : fast_launch_t<dl_t, true, false, false, CONV>(p, stream, prepare_only);
}

// The fast launches with delta stored as dl_t (bfloat16, or int8 codes).
template <typename dl_t>
cudaError_t fast_launch(const ScanParams& p, int phase1, cudaStream_t stream, bool prepare_only)
{
    return p.conv_w ? fast_launch_c<dl_t, true>(p, phase1, stream, prepare_only)
                    : fast_launch_c<dl_t, false>(p, phase1, stream, prepare_only);
}

}  // namespace

}  // namespace ss
