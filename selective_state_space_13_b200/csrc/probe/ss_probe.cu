// Pipe-throughput probes for the roofline of the scan kernels (measurement only; not part of the
// scan library's ABI).  Each probe runs long chains of independent operations in every lane of
// enough warps to fill every scheduler of every SM, and reports operations per second from CUDA
// events:
//   ss_probe_ffma2  packed fp32 multiply-adds (fma.rn.f32x2), counted per lane element
//   ss_probe_ffma   scalar fp32 multiply-adds
//   ss_probe_ex2    MUFU ex2.approx.ftz.f32
//   ss_probe_issue  warp instructions per second of alternating fp32 multiply-adds and
//                   32-bit integer adds (two pipes: bound by instruction issue)
// Results are written to *ops_per_s; the return value is a cudaError_t.
#include <cuda_runtime.h>

#include <cstdint>

namespace {

constexpr int kIters = 4096;
constexpr int kChains = 8;

__global__ void __launch_bounds__(256) ffma2_kernel(float* out, float seed)
{
    float2 a[kChains];
#pragma unroll
    for (int i = 0; i < kChains; ++i)
        a[i] = make_float2(seed + i + threadIdx.x, seed - i);
    const float2 m = make_float2(0.999f, 1.0001f), c = make_float2(1e-7f, -1e-7f);
    for (int it = 0; it < kIters; ++it)
#pragma unroll
        for (int i = 0; i < kChains; ++i)
            a[i] = __ffma2_rn(a[i], m, c);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kChains; ++i)
        s += a[i].x + a[i].y;
    if (s == 1.2345f)
        out[threadIdx.x] = s;
}

__global__ void __launch_bounds__(256) ffma_kernel(float* out, float seed)
{
    float a[2 * kChains];
#pragma unroll
    for (int i = 0; i < 2 * kChains; ++i)
        a[i] = seed + i + threadIdx.x;
    for (int it = 0; it < kIters; ++it)
#pragma unroll
        for (int i = 0; i < 2 * kChains; ++i)
            a[i] = fmaf(a[i], 0.999f, 1e-7f);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 2 * kChains; ++i)
        s += a[i];
    if (s == 1.2345f)
        out[threadIdx.x] = s;
}

__device__ __forceinline__ float ex2f_approx(float x)
{
    float y;
    asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__global__ void __launch_bounds__(256) ex2_kernel(float* out, float seed)
{
    float a[kChains];
#pragma unroll
    for (int i = 0; i < kChains; ++i)
        a[i] = seed * 1e-3f + i * 1e-4f + threadIdx.x * 1e-6f;
    for (int it = 0; it < kIters / 8; ++it)
#pragma unroll
        for (int i = 0; i < kChains; ++i)
            a[i] = ex2f_approx(a[i]) * -0.5f;  // stays in range; one MUFU op each
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kChains; ++i)
        s += a[i];
    if (s == 1.2345f)
        out[threadIdx.x] = s;
}

// Independent fp32 multiply-adds and 32-bit integer adds, alternating: two pipes, so the rate is
// bound by instruction issue (one warp instruction per clock per scheduler) rather than by one
// pipe.
__global__ void __launch_bounds__(256) issue_kernel(float* out, int seed)
{
    float f[kChains];
    int a[kChains];
#pragma unroll
    for (int i = 0; i < kChains; ++i) {
        f[i] = seed + i + threadIdx.x;
        a[i] = seed + i * 7 + threadIdx.x;
    }
    for (int it = 0; it < kIters; ++it)
#pragma unroll
        for (int i = 0; i < kChains; ++i) {
            f[i] = fmaf(f[i], 0.999f, 1e-7f);
            asm volatile("add.u32 %0, %0, %1;" : "+r"(a[i]) : "r"(it));
        }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kChains; ++i)
        s += f[i] + static_cast<float>(a[i]);
    if (s == 1.2345f)
        out[threadIdx.x] = s;
}

template <typename Launch>
cudaError_t time_it(Launch launch, double ops_per_launch, double* ops_per_s)
{
    cudaEvent_t a, b;
    cudaError_t e = cudaEventCreate(&a);
    if (e != cudaSuccess)
        return e;
    if ((e = cudaEventCreate(&b)) != cudaSuccess) {
        cudaEventDestroy(a);
        return e;
    }
    launch();  // warm-up
    float best = 1e30f;
    for (int rep = 0; rep < 5 && e == cudaSuccess; ++rep) {
        cudaEventRecord(a);
        launch();
        cudaEventRecord(b);
        e = cudaEventSynchronize(b);
        float ms = 0.f;
        if (e == cudaSuccess && (e = cudaEventElapsedTime(&ms, a, b)) == cudaSuccess && ms < best)
            best = ms;
    }
    if (e == cudaSuccess)
        e = cudaGetLastError();
    cudaEventDestroy(a);
    cudaEventDestroy(b);
    *ops_per_s = ops_per_launch / (best * 1e-3);
    return e;
}

int blocks()
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms * 8;  // 8 blocks of 8 warps per SM
}

float* scratch()
{
    static float* p = nullptr;
    if (!p && cudaMalloc(&p, 1024 * sizeof(float)) != cudaSuccess)
        p = nullptr;
    return p;
}

}  // namespace

extern "C" {

int ss_probe_ffma2(double* ops_per_s)
{
    const int nb = blocks();
    float* out = scratch();
    const double ops = 2.0 * kChains * kIters * 256.0 * nb;  // lane elements
    return time_it([&] { ffma2_kernel<<<nb, 256>>>(out, 1.f); }, ops, ops_per_s);
}

int ss_probe_ffma(double* ops_per_s)
{
    const int nb = blocks();
    float* out = scratch();
    const double ops = 2.0 * kChains * kIters * 256.0 * nb;
    return time_it([&] { ffma_kernel<<<nb, 256>>>(out, 1.f); }, ops, ops_per_s);
}

int ss_probe_ex2(double* ops_per_s)
{
    const int nb = blocks();
    float* out = scratch();
    const double ops = 1.0 * kChains * (kIters / 8) * 256.0 * nb;
    return time_it([&] { ex2_kernel<<<nb, 256>>>(out, 1.f); }, ops, ops_per_s);
}

int ss_probe_issue(double* warp_inst_per_s)
{
    const int nb = blocks();
    float* out = scratch();
    const double ops = 2.0 * kChains * kIters * (256.0 / 32.0) * nb;  // warp instructions
    return time_it([&] { issue_kernel<<<nb, 256>>>(out, 1); }, ops, warp_inst_per_s);
}

}  // extern "C"
