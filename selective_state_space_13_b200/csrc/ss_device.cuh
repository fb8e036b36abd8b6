// Device helpers of the scan and merge kernels: PTX wrappers for mbarriers, bulk and tensor-map
// copies and programmatic dependent launch, the MUFU approximations the fast arithmetic uses,
// the index map of the scan orders, and the host-side tensor-map encoding and launch helper.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ss_internal.h"

namespace ss {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kTinyW = 5.421010862427522e-20f;  // 2^-64
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s
constexpr unsigned long long kTestWaitNs = 20000000ull;     // 20 ms (test hook)
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

// Tiled tensor copies global -> shared through a tensor map (a __grid_constant__ parameter);
// coordinates are in elements, innermost first.
__device__ __forceinline__ void tma_2d(void* dst, const CUtensorMap* map, int32_t c0, int32_t c1,
                                       uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_3d(void* dst, const CUtensorMap* map, int32_t c0, int32_t c1,
                                       int32_t c2, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start (launch_dependents);
// wait until the previous kernel has finished and its writes are visible (wait).
__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
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

__device__ __forceinline__ float tanh_approx(float x)
{
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

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

// ---------------------------------------------------------------------------- host helpers

// Launch `kern(p)`; with `dependent`, the launch may begin before the previous kernel in the
// stream has finished (programmatic dependent launch).
template <typename Kern, typename P>
cudaError_t launch_ex(Kern kern, unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                      bool dependent, const P& p)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

// cuTensorMapEncodeTiled, looked up once through the runtime (no link-time libcuda dependency).
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

// A row-major tensor of `rank` dims (innermost first) with element strides `pitch` bytes for
// dims 1.., read in boxes `box`; out-of-range elements read as zero.
template <typename T> constexpr CUtensorMapDataType map_type()
{
    return sizeof(T) == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8  // int8 codes, reinterpreted in the kernel
           : sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                            : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
}

inline bool encode(CUtensorMap* map, const void* base, CUtensorMapDataType type, int rank,
                   const cuuint64_t* dims, const cuuint64_t* pitch, const cuuint32_t* box)
{
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn)
        return false;
    const cuuint32_t unit[3] = {1, 1, 1};
    return fn(map, type,
              static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, pitch, box, unit,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tensor maps of u, z and delta for boxes of `box_ch` channels x kTile rows (2D, row orders)
// and box_ch channels x 1 x 8 image rows (3D, column orders with H % 8 == 0).
template <typename io_t, typename dl_t>
cudaError_t make_maps(ScanParams& p, bool need_z, int box_ch)
{
    constexpr CUtensorMapDataType ty = map_type<io_t>();
    constexpr CUtensorMapDataType ty_dl = map_type<dl_t>();
    const cuuint64_t esz = sizeof(io_t);
    const cuuint64_t D = static_cast<cuuint64_t>(p.D);
    const cuuint32_t box2[2] = {static_cast<cuuint32_t>(box_ch), static_cast<cuuint32_t>(kTile)};
    const cuuint64_t pitch2[1] = {D * esz};
    const cuuint64_t dims_bl[2] = {D, static_cast<cuuint64_t>(p.batch * p.L)};
    const cuuint64_t dims_kbl[2] = {D, static_cast<cuuint64_t>(p.K * p.batch * p.L)};
    const int64_t u_blocks = p.u_per_dir ? p.K * p.batch : p.batch;  // row blocks of u
    const cuuint64_t dims_u[2] = {D, static_cast<cuuint64_t>(u_blocks * p.L)};
    const cuuint64_t pitch_dl[1] = {D * sizeof(dl_t)};
    if (!encode(&p.tm_u, p.u, ty, 2, dims_u, pitch2, box2) ||
        !encode(&p.tm_dl, p.delta, ty_dl, 2, dims_kbl, pitch_dl, box2) ||
        (need_z && !encode(&p.tm_z, p.z, ty, 2, dims_bl, pitch2, box2)))
        return cudaErrorInvalidValue;
    bool col = false;
    for (int k = 0; k < p.K; ++k)
        col = col || p.dirs[k] == SS_DIR_COL || p.dirs[k] == SS_DIR_COL_REV;
    p.col3d = (col && p.H > 0 && p.H % 8 == 0) ? 1 : 0;
    if (p.col3d) {
        const cuuint32_t box3[3] = {static_cast<cuuint32_t>(box_ch), 1, 8};
        const cuuint64_t pitch3[2] = {D * esz, static_cast<cuuint64_t>(p.W) * D * esz};
        const cuuint64_t dims3[3] = {D, static_cast<cuuint64_t>(p.W),
                                     static_cast<cuuint64_t>(p.batch * p.H)};
        const cuuint64_t dims3u[3] = {D, static_cast<cuuint64_t>(p.W),
                                      static_cast<cuuint64_t>(u_blocks * p.H)};
        if (!encode(&p.tm_u3, p.u, ty, 3, dims3u, pitch3, box3) ||
            (need_z && !encode(&p.tm_z3, p.z, ty, 3, dims3, pitch3, box3)))
            return cudaErrorInvalidValue;
    }
    return cudaSuccess;
}

}  // namespace

}  // namespace ss
