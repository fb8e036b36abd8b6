// Internal declarations shared by the host entry points (ss_api.cu) and the kernels (ss_scan.cu).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "selective_scan.h"

namespace ss {

// Steps per pipeline stage of the shared-memory ring.
constexpr int kTile = 16;
// Rows whose per-step scalars the fast path computes together.
constexpr int kGroup = 8;

// Everything a scan launch needs.  Device pointers are the caller's; nothing here is owned.
// The tensor maps are filled in by prepare_scan.
struct ScanParams {
    CUtensorMap tm_u, tm_z;    // u, z as [batch*L rows, D]: boxes of kTile rows x DC channels
    CUtensorMap tm_dl;         // delta as [K*batch*L rows, D], same boxes
    CUtensorMap tm_u3, tm_z3;  // u, z as [batch*H, W, D]: boxes of 8 image rows of one column
    const void* u;          // [batch, L, D] io, spatial order ([K, batch, L, D] with u_per_dir)
    const void* delta;      // [K, batch, L, D] io (or int8 codes), scan order
    const float* A;         // [D, N] ([K, D, N] with params_per_dir)
    const void* B;          // [K, batch, L, N] io, scan order
    const void* C;          // [K, batch, L, N] io, scan order
    const float* Dskip;     // [D] ([K, D] with params_per_dir) or null
    const void* z;          // [batch, L, D] io or null
    const float* bias;      // [D] ([K, D] with params_per_dir) or null
    void* out;              // [batch, L, D] io (single direction) or null
    float* ypart;           // [K, batch, L, D] fp32 per-direction outputs (several directions)
    float* last_state;      // [K, batch, D, N] or null
    const float* init_state;  // [K, batch, D, N] state before step 0, or null (zero)
    const float* conv_w;    // [K, D, conv_width] causal conv taps per direction, or null
    const float* conv_b;    // [K, D] conv bias, or null (zero)
    const float* delta_scale;  // [D] scale of int8 delta codes, or null (delta in io type)
    // segment carries: fp32 for bf16 io, fp64 for fp32 io (read through the kernels' state type)
    float* carry_h;         // [K, batch, S, D, N] end state of each segment scanned from zero
    float* carry_s;         // [K, batch, S, D] sum over the segment of Delta (times log2(e) in fp32)
    int64_t batch, L, D;
    int64_t seg_len;        // steps per segment (last segment may be shorter)
    int32_t N, K, S;
    int32_t dirs[SS_MAX_DIRS];
    int32_t H, W;
    int32_t softplus;
    int32_t force_generic;  // 1: never take the A[d,n] = (n+1) A[d,0] shortcut
    int32_t col3d;          // 1: column orders load through tm_u3 / tm_z3 (H % 8 == 0)
    int32_t zoh;            // 1: Bbar = (exp(Delta*A) - 1) / A * B (precise arithmetic)
    int32_t test_timeout;   // 1: test hook, wait on a barrier nothing completes and report
    int32_t conv_width;     // taps of conv_w (1..SS_MAX_CONV_WIDTH) when conv_w is set
    int32_t u_per_dir;      // 1: direction k reads its own input u[k]
    int32_t params_per_dir; // 1: direction k reads its own A[k], Dskip[k], bias[k]
    unsigned int* status;   // the device error word (status_word()), or'ed by bounded waits
};

struct MergeParams {
    const float* ypart;     // [K, batch, L, D]
    const void* z;          // [batch, L, D] io or null
    void* out;              // [batch, L, D] io
    int64_t rows;           // batch * L
    int64_t D;
    int32_t K;
};

// Channels handled by one CTA of the scan kernel.
int channels_per_cta();

// Device address of the library's error word on the current device (looked up once per device),
// or null if the runtime fails.
unsigned int* status_word();

// The scan launches, one translation unit per io type and delta storage (bfloat16 io with delta
// as bfloat16 or int8 codes, fp32 io).  phase1 = 1: segment aggregates only (segments 0..S-2);
// phase1 = 0: the scan of all S segments.  With prepare_only nothing is launched: only the
// kernel's shared-memory attribute is set.
cudaError_t scan_launch_f32(const ScanParams& p, int phase1, cudaStream_t stream, bool prepare_only);
cudaError_t scan_launch_bf16(const ScanParams& p, int phase1, cudaStream_t stream, bool prepare_only);
cudaError_t scan_launch_bf16_i8(const ScanParams& p, int phase1, cudaStream_t stream,
                                bool prepare_only);

// Everything a call needs before its first launch: the tensor maps of u, z and delta encoded into
// p, and the shared-memory attributes of every kernel the call launches.  Nothing is launched,
// so a failure here leaves the stream untouched.
cudaError_t prepare_scan(ScanParams& p, int io_dtype);

// Enqueue one scan launch (phase1 as above) with the tensor maps prepare_scan encoded.
cudaError_t launch_scan(const ScanParams& p, int io_dtype, int phase1, cudaStream_t stream);

// Enqueue the direction merge + gate: out = (sum_k ypart[k]) * silu(z).
cudaError_t launch_merge(const MergeParams& p, int io_dtype, cudaStream_t stream);

// Same index function the kernels use (host copy of the device function).
int64_t position_host(int32_t dir, int64_t L, int32_t H, int32_t W, int64_t t);

// Synchronise `stream`, read this library's device error word on the current device into *value,
// and reset it when `clear` is set.
cudaError_t read_status(cudaStream_t stream, bool clear, unsigned int* value);

}  // namespace ss
