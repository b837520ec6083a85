// fp8fg.cu -- C ABI of the library (declared in include/fp8fg.h): argument
// validation, per-device capability checks, TMA descriptor encoding and
// kernel launches.  Single translation unit: the kernels and the device
// error word live in the headers included below.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "../../include/fp8fg.h"
#include "gemm_kernels.cuh"
#include "gemm_pair_kernels.cuh"
#include "quant_kernels.cuh"
#include "quant_stream_kernels.cuh"
#include "dequant_kernels.cuh"
#include "quant_gather_kernels.cuh"
#include "quant_act_kernels.cuh"
#include "quant_weight_kernels.cuh"

namespace fp8fg {
namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    std::atomic<int> state{0};  // 0 unknown, 1 ok, 2 unsupported
    int num_sms = 0;
    int max_pairs = 0;          // co-resident 2-CTA clusters of the pair GEMM
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Current device must be compute capability 10.0 (B200, sm_100a code).
fp8_status_t current_device(int* dev_out, int* sms_out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return FP8_ERR_DEVICE;
    }
    DeviceInfo& d = g_dev[dev];
    int st = d.state.load(std::memory_order_acquire);
    if (st == 0) {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        st = d.state.load(std::memory_order_relaxed);
        if (st == 0) {
            int major = 0, minor = 0, sms = 0;
            if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
                cudaGetLastError();
                return FP8_ERR_CUDA;
            }
            bool ok = (major == 10 && minor == 0);
            if (ok) {
                // Opt the GEMM kernels into their shared-memory footprint.
                const void* kernels[] = {
                    reinterpret_cast<const void*>(&blockscaled_gemm_kernel<false, false>),
                    reinterpret_cast<const void*>(&blockscaled_gemm_kernel<false, true>),
                    reinterpret_cast<const void*>(&blockscaled_gemm_kernel<true, false>),
                    reinterpret_cast<const void*>(&blockscaled_gemm_kernel<true, true>)};
                for (const void* k : kernels) {
                    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kGemmSmemBytes)) != cudaSuccess) {
                        cudaGetLastError();
                        return FP8_ERR_CUDA;
                    }
                }
                const void* pair_kernels[] = {
                    reinterpret_cast<const void*>(&blockscaled_gemm_pair_kernel<false, false>),
                    reinterpret_cast<const void*>(&blockscaled_gemm_pair_kernel<false, true>),
                    reinterpret_cast<const void*>(&blockscaled_gemm_pair_kernel<true, false>),
                    reinterpret_cast<const void*>(&blockscaled_gemm_pair_kernel<true, true>),
                    reinterpret_cast<const void*>(&blockscaled_gemm_pair_kernel<false, true, true>),
                    reinterpret_cast<const void*>(&blockscaled_gemm_pair_kernel<false, false, false, true>),
                    reinterpret_cast<const void*>(&blockscaled_gemm_pair_kernel<false, true, false, true>)};
                for (int i = 0; i < 7; ++i) {
                    const size_t bytes = (i == 2 || i == 3) ? kGemmPairGroupedSmemBytes
                                         : i >= 5           ? kGemmPairColScaleSmemBytes
                                                            : kGemmPairSmemBytes;
                    if (cudaFuncSetAttribute(pair_kernels[i],
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(bytes)) != cudaSuccess) {
                        cudaGetLastError();
                        return FP8_ERR_CUDA;
                    }
                }
                const void* qa_kernels[] = {
                    reinterpret_cast<const void*>(&quant_act_rows_kernel<kRowsPlain>),
                    reinterpret_cast<const void*>(&quant_act_rows_kernel<kRowsScatter>),
                    reinterpret_cast<const void*>(&quant_weight_rows_kernel<kQwBlockRows>),
                    reinterpret_cast<const void*>(&quant_weight_rows_kernel<kQwBlockCols>),
                    reinterpret_cast<const void*>(&quant_weight_rows_kernel<kQwColTiles>)};
                const size_t qa_bytes[] = {kQaSmemBytes, kQaSmemBytes, kQwSmemBytes,
                                           kQwSmemBytes, kQwSmemBytes};
                for (int i = 0; i < 5; ++i) {
                    if (cudaFuncSetAttribute(qa_kernels[i],
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(qa_bytes[i])) != cudaSuccess) {
                        cudaGetLastError();
                        return FP8_ERR_CUDA;
                    }
                }
                const void* qs_kernels[] = {
                    reinterpret_cast<const void*>(&quant_stream_kernel<uint16_t, kQuantAct>),
                    reinterpret_cast<const void*>(&quant_stream_kernel<uint16_t, kQuantWeight>),
                    reinterpret_cast<const void*>(&quant_stream_kernel<uint16_t, kQuantWeightT>),
                    reinterpret_cast<const void*>(&quant_stream_kernel<float, kQuantAct>),
                    reinterpret_cast<const void*>(&quant_stream_kernel<float, kQuantWeight>),
                    reinterpret_cast<const void*>(&quant_stream_kernel<float, kQuantWeightT>),
                    reinterpret_cast<const void*>(&quant_stream_kernel<uint16_t, kQuantActT>)};
                const size_t qs_bytes[] = {quant_stream_smem_bytes<uint16_t, kQuantAct>(),
                                           quant_stream_smem_bytes<uint16_t, kQuantWeight>(),
                                           quant_stream_smem_bytes<uint16_t, kQuantWeightT>(),
                                           quant_stream_smem_bytes<float, kQuantAct>(),
                                           quant_stream_smem_bytes<float, kQuantWeight>(),
                                           quant_stream_smem_bytes<float, kQuantWeightT>(),
                                           quant_stream_smem_bytes<uint16_t, kQuantActT>()};
                for (int i = 0; i < 7; ++i) {
                    if (cudaFuncSetAttribute(qs_kernels[i],
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(qs_bytes[i])) != cudaSuccess) {
                        cudaGetLastError();
                        return FP8_ERR_CUDA;
                    }
                }
                // CTA pairs that can be resident at once (a cluster must fit in
                // one GPC): the persistent grid must not exceed it, or the
                // surplus pairs would run as a second wave.
                cudaLaunchConfig_t cfg = {};
                cfg.gridDim = dim3(2, 1, 1);
                cfg.blockDim = dim3(kGemmThreads, 1, 1);
                cfg.dynamicSmemBytes = kGemmPairSmemBytes;
                cudaLaunchAttribute attr[1];
                attr[0].id = cudaLaunchAttributeClusterDimension;
                attr[0].val.clusterDim.x = 2;
                attr[0].val.clusterDim.y = 1;
                attr[0].val.clusterDim.z = 1;
                cfg.attrs = attr;
                cfg.numAttrs = 1;
                int clusters = 0;
                if (cudaOccupancyMaxActiveClusters(&clusters,
                                                   blockscaled_gemm_pair_kernel<false, true>,
                                                   &cfg) != cudaSuccess ||
                    clusters < 1) {
                    cudaGetLastError();
                    return FP8_ERR_CUDA;
                }
                d.max_pairs = clusters;
            }
            d.num_sms = sms;
            st = ok ? 1 : 2;
            d.state.store(st, std::memory_order_release);
        }
    }
    if (st != 1) return FP8_ERR_DEVICE;
    *dev_out = dev;
    *sms_out = d.num_sms;
    return FP8_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        else
            cudaGetLastError();
    });
    return g_encode;
}

// 2-D uint8 tensor [rows, cols] with row stride `ld` bytes, box
// [box_rows, 128 bytes], 128-byte swizzle, zero fill out of bounds.
bool make_operand_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                      uint64_t ld, uint32_t box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

inline fp8_status_t launch_status() {
    return cudaGetLastError() == cudaSuccess ? FP8_OK : FP8_ERR_CUDA;
}

// Grouped GEMM: for contractions of at least this many K, the CTA-pair
// kernel (256-row tiles) takes each group's whole 256-row blocks and a
// remainder of more than 128 rows, and the one-CTA kernel a remainder of
// 1-128 rows; shorter contractions run on the one-CTA kernel alone
// (128-row tiles).
constexpr int64_t kGroupedPairMinK = 4096;

// L2 bytes one raster band of the dense GEMM may hold (of the B200's 126 MB;
// the rest serves the streamed operand's chunks and the output).
constexpr int64_t kL2BandBytes = int64_t{72} << 20;

int elem_size_in(fp8_in_t t) { return t == FP8_IN_BF16 ? 2 : (t == FP8_IN_FP32 ? 4 : 0); }
int elem_size_out(fp8_out_t t) { return t == FP8_OUT_BF16 ? 2 : (t == FP8_OUT_FP32 ? 4 : 0); }

// Grid of resident-sized blocks, a multiple of the SM count.
int64_t grid_for(int64_t work_blocks, int sms, int blocks_per_sm) {
    const int64_t cap = static_cast<int64_t>(sms) * blocks_per_sm;
    return work_blocks < cap ? work_blocks : cap;
}

// K == 0: the product is empty, C = 0.  Only c is used.
fp8_status_t zero_output(void* c, fp8_out_t ct, int64_t ldc, int64_t rows, int64_t cols,
                         cudaStream_t stream) {
    const int oes = elem_size_out(ct);
    if (!c) return FP8_ERR_NULL;
    if (ldc < cols) return FP8_ERR_LAYOUT;
    if (!aligned16(c) || (ldc * oes) % 16 != 0) return FP8_ERR_ALIGN;
    int dev, sms;
    fp8_status_t st = current_device(&dev, &sms);
    if (st != FP8_OK) return st;
    const int64_t grid = grid_for((rows * cols + 255) / 256, sms, 8);
    if (ct == FP8_OUT_BF16)
        zero_rows_kernel<__nv_bfloat16><<<static_cast<unsigned>(grid), 256, 0, stream>>>(
            static_cast<__nv_bfloat16*>(c), rows, cols, ldc);
    else
        zero_rows_kernel<float><<<static_cast<unsigned>(grid), 256, 0, stream>>>(
            static_cast<float*>(c), rows, cols, ldc);
    return launch_status();
}


// 2-D input tensor [rows, cols] (bf16 or fp32) with row stride `ld`
// elements, box 128 x 128, no swizzle, zero fill out of bounds.
bool make_input_map(CUtensorMap* map, const void* base, fp8_in_t t, uint64_t rows, uint64_t cols,
                    uint64_t ld) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const int es = elem_size_in(t);
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * static_cast<uint64_t>(es)};
    cuuint32_t box[2] = {128, 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, t == FP8_IN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                           : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                     2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// bf16 activations [M, K] (row stride ld elements) for the row kernel:
// boxes of 32 rows x 64 columns, 128-byte swizzle, zero fill out of bounds.
bool make_act_rows_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint64_t ld) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kQaRows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 128x128 quantization of a bf16 weight [K, N], one block row per thread
// (quant_weight_rows_kernel): boxes of 128 rows x 64 columns, 128-byte
// swizzle; one persistent CTA of kQwGroups groups per SM.
// mode kQwColTiles: 128x1 tiles of x [K rows, N columns] (the tokens are the
// rows), codes transposed, s[column * sb_stride_nb + band * sb_stride_kb].
fp8_status_t launch_quant_weight_rows(const void* w, int64_t K, int64_t N, int64_t ldw,
                                      uint8_t* q, int mode, int64_t ldq, float* sb,
                                      int64_t sb_stride_kb, int64_t sb_stride_nb, int sms,
                                      cudaStream_t stream) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return FP8_ERR_CUDA;
    CUtensorMap map;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(K)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldw) * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(w), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return FP8_ERR_CUDA;
    QwParams p{};
    p.nbr = K / 128;
    p.nbc = N / 128;
    p.nblocks = p.nbr * p.nbc;
    p.q = q; p.ldq = ldq;
    p.s = sb; p.s_stride_kb = sb_stride_kb; p.s_stride_nb = sb_stride_nb;
    const int64_t ctas = (p.nblocks + kQwGroups - 1) / kQwGroups;
    const unsigned grid = static_cast<unsigned>(ctas < sms ? ctas : sms);
    if (mode == kQwColTiles)
        quant_weight_rows_kernel<kQwColTiles><<<grid, kQwThreads, kQwSmemBytes, stream>>>(map, p);
    else if (mode == kQwBlockCols)
        quant_weight_rows_kernel<kQwBlockCols><<<grid, kQwThreads, kQwSmemBytes, stream>>>(map, p);
    else
        quant_weight_rows_kernel<kQwBlockRows><<<grid, kQwThreads, kQwSmemBytes, stream>>>(map, p);
    return launch_status();
}

// 1x128 quantization of bf16 rows, one row per thread (quant_act_rows_kernel):
// one persistent CTA of kQaWarps independent warps per SM.
// With `dest` (scatter form): input row t goes to the output rows
// dest[t * topk + j] (of out_rows); otherwise row m goes to row m.
fp8_status_t launch_quant_act_rows(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                                   int64_t ldq, float* sa, int64_t sa_stride_m,
                                   int64_t sa_stride_kb, int sms, cudaStream_t stream,
                                   const int32_t* dest = nullptr, int64_t topk = 0,
                                   int64_t out_rows = 0) {
    CUtensorMap map;
    if (!make_act_rows_map(&map, x, static_cast<uint64_t>(M), static_cast<uint64_t>(K),
                           static_cast<uint64_t>(ldx)))
        return FP8_ERR_CUDA;
    QaParams p{};
    p.rows = M;
    p.nkb = K / 128;
    p.nboxes = ((M + kQaRows - 1) / kQaRows) * p.nkb;
    p.q = q; p.ldq = ldq;
    p.s = sa; p.s_stride_m = sa_stride_m; p.s_stride_kb = sa_stride_kb;
    p.dest = dest; p.topk = topk; p.out_rows = out_rows;
    const int64_t ctas = (p.nboxes + kQaWarps - 1) / kQaWarps;
    const unsigned grid = static_cast<unsigned>(ctas < sms ? ctas : sms);
    if (dest)
        quant_act_rows_kernel<kRowsScatter><<<grid, kQaThreads, kQaSmemBytes, stream>>>(map, p);
    else
        quant_act_rows_kernel<kRowsPlain><<<grid, kQaThreads, kQaSmemBytes, stream>>>(map, p);
    return launch_status();
}

template <typename T, int kMode>
fp8_status_t launch_quant_stream_t(const CUtensorMap& map, const QsParams& p, int sms,
                                   cudaStream_t stream) {
    const int64_t boxes = p.nbr * p.nbc;
    const unsigned grid = static_cast<unsigned>(boxes < sms ? boxes : sms);
    QsParams q = p;
    const int64_t step = static_cast<int64_t>(kQsGroups) * grid;
    q.step_r = step / p.nbc;
    q.step_c = step - q.step_r * p.nbc;
    quant_stream_kernel<T, kMode>
        <<<grid, kQsThreads, quant_stream_smem_bytes<T, kMode>(), stream>>>(map, q);
    return launch_status();
}

// One persistent CTA per SM streams the 128x128 boxes of the input.
fp8_status_t launch_quant_stream(const void* in, fp8_in_t t, int64_t ld, const QsParams& p,
                                 int mode, int sms, cudaStream_t stream) {
    CUtensorMap map;
    if (!make_input_map(&map, in, t, static_cast<uint64_t>(p.rows), static_cast<uint64_t>(p.cols),
                        static_cast<uint64_t>(ld)))
        return FP8_ERR_CUDA;
    if (t == FP8_IN_BF16) {
        if (mode == kQuantAct) return launch_quant_stream_t<uint16_t, kQuantAct>(map, p, sms, stream);
        if (mode == kQuantActT)
            return launch_quant_stream_t<uint16_t, kQuantActT>(map, p, sms, stream);
        if (mode == kQuantWeight)
            return launch_quant_stream_t<uint16_t, kQuantWeight>(map, p, sms, stream);
        return launch_quant_stream_t<uint16_t, kQuantWeightT>(map, p, sms, stream);
    }
    if (mode == kQuantAct) return launch_quant_stream_t<float, kQuantAct>(map, p, sms, stream);
    if (mode == kQuantWeight) return launch_quant_stream_t<float, kQuantWeight>(map, p, sms, stream);
    return launch_quant_stream_t<float, kQuantWeightT>(map, p, sms, stream);
}

// Persistent CTA-pair GEMM: `pairs` clusters of 2 CTAs.
template <bool kGrouped, bool kQuantOut = false, bool kColScaleB = false>
fp8_status_t launch_pair_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmParams& p,
                              int64_t pairs, fp8_out_t c_type, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = kGrouped     ? kGemmPairGroupedSmemBytes
                           : kColScaleB ? kGemmPairColScaleSmemBytes
                                        : kGemmPairSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (kColScaleB && !kGrouped && c_type == FP8_OUT_BF16)
        e = cudaLaunchKernelEx(&cfg, blockscaled_gemm_pair_kernel<false, true, false, true>, tmA, tmB, p);
    else if (kColScaleB && !kGrouped)
        e = cudaLaunchKernelEx(&cfg, blockscaled_gemm_pair_kernel<false, false, false, true>, tmA, tmB, p);
    else if (kQuantOut)
        e = cudaLaunchKernelEx(&cfg, blockscaled_gemm_pair_kernel<kGrouped, true, true>, tmA, tmB, p);
    else if (c_type == FP8_OUT_BF16)
        e = cudaLaunchKernelEx(&cfg, blockscaled_gemm_pair_kernel<kGrouped, true>, tmA, tmB, p);
    else
        e = cudaLaunchKernelEx(&cfg, blockscaled_gemm_pair_kernel<kGrouped, false>, tmA, tmB, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return FP8_ERR_CUDA;
    }
    return launch_status();
}

// Dense GEMM on CTA pairs after the argument checks; `out` carries the
// output fields (c / ldc, or the quantized-output fields).
template <bool kQuantOut, bool kColScaleB = false>
fp8_status_t dense_gemm(const uint8_t* a, int64_t lda, const float* sa, int64_t sa_stride_m,
                        int64_t sa_stride_kb, const uint8_t* b, int64_t ldb, const float* sb,
                        int64_t sb_stride_kb, int64_t sb_stride_nb, const GemmParams& out,
                        fp8_out_t c_type, int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
    // 256 x 256 tiles, one per CTA pair (two SMs).
    const int64_t num_mt = (M + kPairBM - 1) / kPairBM, num_nt = (N + kBN - 1) / kBN;
    if (num_mt * num_nt > INT32_MAX || M > INT32_MAX) return FP8_ERR_SHAPE;
    int dev, sms;
    fp8_status_t st = current_device(&dev, &sms);
    if (st != FP8_OK) return st;

    CUtensorMap tmA, tmB;
    const uint64_t kcols = static_cast<uint64_t>(K);
    if (!make_operand_map(&tmA, a, static_cast<uint64_t>(M), kcols, static_cast<uint64_t>(lda), 128) ||
        !make_operand_map(&tmB, b, static_cast<uint64_t>(N), kcols, static_cast<uint64_t>(ldb), 128))
        return FP8_ERR_CUDA;

    GemmParams p = out;
    p.c_v8 = (p.c != nullptr && aligned32(p.c) &&
              (p.ldc * elem_size_out(c_type)) % 32 == 0) ? 1 : 0;
    p.qc_v8 = (p.qc != nullptr && aligned32(p.qc) && p.ldqc % 32 == 0) ? 1 : 0;
    p.sa = sa; p.sa_sm = sa_stride_m; p.sa_skb = sa_stride_kb;
    p.sb = sb; p.sb_sg = 0; p.sb_skb = sb_stride_kb; p.sb_snb = sb_stride_nb;
    p.M = M; p.N = N;
    p.nkb = static_cast<int>(K / 128);
    p.num_mt = static_cast<int>(num_mt);
    p.num_nt = static_cast<int>(num_nt);
    // Tile raster for L2 reuse.  The smaller operand is cut into bands that
    // stay in L2 (at most kL2BandBytes of the 126 MB) while the pairs walk
    // across the larger one: the band operand is read from HBM once, the
    // streamed one once per band.  Bands are balanced (equal tile counts).
    const int64_t a_bytes = num_mt * static_cast<int64_t>(kPairBM) * K;
    const int64_t b_bytes = num_nt * static_cast<int64_t>(kBN) * K;
    const bool band_over_n = b_bytes < a_bytes;
    const int64_t tiles = band_over_n ? num_nt : num_mt;
    const int64_t panel = (band_over_n ? kBN : kPairBM) * K;     // bytes of one tile's panel
    int64_t nbands = (tiles * panel + kL2BandBytes - 1) / kL2BandBytes;
    nbands = nbands < 1 ? 1 : (nbands > tiles ? tiles : nbands);
    const int band = static_cast<int>((tiles + nbands - 1) / nbands);
    p.band_m = band_over_n ? 1 : band;
    p.band_n = band_over_n ? band : 0;
    p.offsets = nullptr; p.G = 1;
    const int64_t pairs = grid_for(num_mt * num_nt, g_dev[dev].max_pairs, 1);
    return launch_pair_gemm<false, kQuantOut, kColScaleB>(tmA, tmB, p, pairs, c_type, stream);
}

}  // namespace
}  // namespace fp8fg

using namespace fp8fg;

extern "C" {

fp8_status_t fp8_quantize_act_1x128_gather(const void* x, fp8_in_t x_type, int64_t src_rows,
                                           int64_t K, int64_t ldx, const int32_t* rows,
                                           int64_t R, uint8_t* q, int64_t ldq, float* sa,
                                           int64_t sa_stride_m, int64_t sa_stride_kb,
                                           fp8_stream_t stream) {
    const int es = elem_size_in(x_type);
    if (es == 0) return FP8_ERR_DTYPE;
    if (src_rows < 0 || R < 0 || K < 0 || K % 128 != 0) return FP8_ERR_SHAPE;
    if (R == 0 || K == 0) return FP8_OK;
    if (!x || !rows || !q || !sa) return FP8_ERR_NULL;
    if (ldx < K || ldq < K || sa_stride_m < 0 || sa_stride_kb < 0) return FP8_ERR_LAYOUT;
    if (!aligned16(x) || (ldx * es) % 16 != 0 || !aligned16(q) || ldq % 16 != 0 ||
        !aligned4(sa) || !aligned4(rows))
        return FP8_ERR_ALIGN;
    int dev, sms;
    fp8_status_t st = current_device(&dev, &sms);
    if (st != FP8_OK) return st;
    // one half-warp per output row at a time
    const int64_t grid = grid_for((R + 15) / 16, sms, kGqMinBlocks);
    const unsigned g = static_cast<unsigned>(grid);
    const int64_t nkb = K / 128;
    if (x_type == FP8_IN_BF16)
        quant_gather_kernel<uint16_t><<<g, kGqThreads, 0, stream>>>(
            static_cast<const uint16_t*>(x), src_rows, ldx, rows, R, nkb, q, ldq, sa, sa_stride_m,
            sa_stride_kb);
    else
        quant_gather_kernel<float><<<g, kGqThreads, 0, stream>>>(
            static_cast<const float*>(x), src_rows, ldx, rows, R, nkb, q, ldq, sa, sa_stride_m,
            sa_stride_kb);
    return launch_status();
}

fp8_status_t fp8_quantize_act_1x128_scatter(const void* x, fp8_in_t x_type, int64_t T, int64_t K,
                                            int64_t ldx, const int32_t* dest, int64_t topk,
                                            uint8_t* q, int64_t R, int64_t ldq, float* sa,
                                            int64_t sa_stride_m, int64_t sa_stride_kb,
                                            fp8_stream_t stream) {
    const int es = elem_size_in(x_type);
    if (es == 0) return FP8_ERR_DTYPE;
    if (T < 0 || R < 0 || K < 0 || K % 128 != 0 || topk < 0) return FP8_ERR_SHAPE;
    if (T == 0 || K == 0 || topk == 0) return FP8_OK;
    if (x_type != FP8_IN_BF16) return FP8_ERR_DTYPE;
    if (!x || !dest || (R > 0 && (!q || !sa))) return FP8_ERR_NULL;
    if (ldx < K || ldq < K || sa_stride_m < 0 || sa_stride_kb < 0) return FP8_ERR_LAYOUT;
    if (!aligned16(x) || (ldx * es) % 16 != 0 || !aligned4(dest) ||
        (R > 0 && (!aligned32(q) || ldq % 32 != 0 || !aligned4(sa))))
        return FP8_ERR_ALIGN;
    if (T > INT32_MAX || R > INT32_MAX || topk > INT32_MAX / (T > 0 ? T : 1)) return FP8_ERR_SHAPE;
    int dev, sms;
    fp8_status_t st = current_device(&dev, &sms);
    if (st != FP8_OK) return st;
    return launch_quant_act_rows(x, T, K, ldx, q, ldq, sa, sa_stride_m, sa_stride_kb, sms, stream,
                                 dest, topk, R);
}

fp8_status_t fp8_dequantize(const uint8_t* q, int64_t rows, int64_t cols, int64_t ldq,
                            const float* s, int64_t s_stride_r, int64_t s_stride_c, int tile_rows,
                            void* out, fp8_out_t out_type, int64_t ldo, fp8_stream_t stream) {
    const int oes = elem_size_out(out_type);
    if (oes == 0) return FP8_ERR_DTYPE;
    if (rows < 0 || cols < 0 || cols % 128 != 0 || (tile_rows != 1 && tile_rows != 128))
        return FP8_ERR_SHAPE;
    if (rows == 0 || cols == 0) return FP8_OK;
    if (!q || !s || !out) return FP8_ERR_NULL;
    if (ldq < cols || ldo < cols || s_stride_r < 0 || s_stride_c < 0) return FP8_ERR_LAYOUT;
    if (!aligned16(q) || ldq % 16 != 0 || !aligned4(s) || !aligned16(out) || (ldo * oes) % 16 != 0)
        return FP8_ERR_ALIGN;
    int dev, sms;
    fp8_status_t st = current_device(&dev, &sms);
    if (st != FP8_OK) return st;
    const int64_t gx = (cols + kDqCodesPerBlock - 1) / kDqCodesPerBlock;
    // kDqBlocksPerSm resident blocks per SM, one wave.
    int64_t gy = (static_cast<int64_t>(sms) * kDqBlocksPerSm + gx - 1) / gx;
    if (gy > rows) gy = rows;
    if (gy > 65535) gy = 65535;
    const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
    const int tile_shift = tile_rows == 128 ? 7 : 0;
    if (out_type == FP8_OUT_BF16)
        dequant_kernel<true><<<grid, kDqThreads, 0, stream>>>(q, rows, cols, ldq, s, s_stride_r,
                                                              s_stride_c, tile_shift, out, ldo);
    else
        dequant_kernel<false><<<grid, kDqThreads, 0, stream>>>(q, rows, cols, ldq, s, s_stride_r,
                                                               s_stride_c, tile_shift, out, ldo);
    return launch_status();
}

const char* fp8_status_string(fp8_status_t s) {
    switch (s) {
        case FP8_OK: return "FP8_OK";
        case FP8_ERR_NULL: return "FP8_ERR_NULL: a required pointer is NULL";
        case FP8_ERR_SHAPE: return "FP8_ERR_SHAPE: bad size (negative, or not a multiple of 128)";
        case FP8_ERR_ALIGN: return "FP8_ERR_ALIGN: pointer or leading dimension not 16-byte aligned";
        case FP8_ERR_LAYOUT: return "FP8_ERR_LAYOUT: unsupported strides or operand orientation";
        case FP8_ERR_DTYPE: return "FP8_ERR_DTYPE: unknown element type";
        case FP8_ERR_DEVICE: return "FP8_ERR_DEVICE: current device is not an sm_100 (B200) GPU";
        case FP8_ERR_CUDA: return "FP8_ERR_CUDA: a CUDA call failed";
        case FP8_ERR_UNIMPLEMENTED: return "FP8_ERR_UNIMPLEMENTED";
        case FP8_ERR_DEVICE_TIMEOUT: return "FP8_ERR_DEVICE_TIMEOUT: a kernel gave up waiting";
    }
    return "unknown fp8_status_t";
}

fp8_status_t fp8_quantize_act_1x128(const void* x, fp8_in_t x_type, int64_t M, int64_t K,
                                    int64_t ldx, uint8_t* q, int64_t ldq, float* sa,
                                    int64_t sa_stride_m, int64_t sa_stride_kb,
                                    fp8_stream_t stream) {
    const int es = elem_size_in(x_type);
    if (es == 0) return FP8_ERR_DTYPE;
    if (M < 0 || K < 0 || K % 128 != 0) return FP8_ERR_SHAPE;
    if (M == 0 || K == 0) return FP8_OK;
    if (!x || !q || !sa) return FP8_ERR_NULL;
    if (ldx < K || ldq < K || sa_stride_m < 0 || sa_stride_kb < 0) return FP8_ERR_LAYOUT;
    if (!aligned16(x) || (ldx * es) % 16 != 0 || !aligned16(q) || ldq % 16 != 0 || !aligned4(sa))
        return FP8_ERR_ALIGN;
    if (M > INT32_MAX) return FP8_ERR_SHAPE;
    int dev, sms;
    fp8_status_t st = current_device(&dev, &sms);
    if (st != FP8_OK) return st;
    // bf16 rows whose codes can leave as 32-byte stores: one row per thread.
    if (x_type == FP8_IN_BF16 && aligned32(q) && ldq % 32 == 0)
        return launch_quant_act_rows(x, M, K, ldx, q, ldq, sa, sa_stride_m, sa_stride_kb, sms,
                                     stream);
    QsParams p{};
    p.rows = M; p.cols = K;
    p.nbr = (M + 127) / 128; p.nbc = K / 128;
    p.q = q; p.ldq = ldq;
    p.s = sa; p.s_stride_r = sa_stride_m; p.s_stride_c = sa_stride_kb;
    return launch_quant_stream(x, x_type, ldx, p, kQuantAct, sms, stream);
}

fp8_status_t fp8_quantize_weight_128x128(const void* w, fp8_in_t w_type, int64_t K, int64_t N,
                                         int64_t ldw, uint8_t* q, int transpose_out,
                                         int64_t ldq, float* sb, int64_t sb_stride_kb,
                                         int64_t sb_stride_nb, fp8_stream_t stream) {
    const int es = elem_size_in(w_type);
    if (es == 0) return FP8_ERR_DTYPE;
    if (K < 0 || N < 0 || K % 128 != 0 || N % 128 != 0) return FP8_ERR_SHAPE;
    if (K == 0 || N == 0) return FP8_OK;
    if (!w || !q || !sb) return FP8_ERR_NULL;
    if (ldw < N || ldq < (transpose_out ? K : N) || sb_stride_kb < 0 || sb_stride_nb < 0)
        return FP8_ERR_LAYOUT;
    if (!aligned16(w) || (ldw * es) % 16 != 0 || !aligned16(q) || ldq % 16 != 0 || !aligned4(sb))
        return FP8_ERR_ALIGN;
    if (K > INT32_MAX || N > INT32_MAX) return FP8_ERR_SHAPE;
    int dev, sms;
    fp8_status_t st = current_device(&dev, &sms);
    if (st != FP8_OK) return st;
    // bf16 weights whose codes can leave as 32-byte stores: one block row per
    // thread.
    if (w_type == FP8_IN_BF16 && aligned32(q) && ldq % 32 == 0)
        return launch_quant_weight_rows(w, K, N, ldw, q, transpose_out ? kQwBlockCols : kQwBlockRows,
                                        ldq, sb, sb_stride_kb, sb_stride_nb, sms, stream);
    QsParams p{};
    p.rows = K; p.cols = N;
    p.nbr = K / 128; p.nbc = N / 128;
    p.q = q; p.ldq = ldq;
    p.s = sb; p.s_stride_r = sb_stride_kb; p.s_stride_c = sb_stride_nb;
    return launch_quant_stream(w, w_type, ldw, p, transpose_out ? kQuantWeightT : kQuantWeight,
                               sms, stream);
}

static fp8_status_t check_gemm_common(const uint8_t* a, int64_t lda, const float* sa,
                                      int64_t sa_sm, int64_t sa_skb, const uint8_t* b, int64_t ldb,
                                      const float* sb, int64_t sb_skb, int64_t sb_snb, void* c,
                                      fp8_out_t ct, int64_t ldc, int64_t N, int64_t K) {
    const int oes = elem_size_out(ct);
    if (oes == 0) return FP8_ERR_DTYPE;
    if (!a || !sa || !b || !sb || !c) return FP8_ERR_NULL;
    if (lda < K || ldb < K || ldc < N || sa_sm < 0 || sa_skb < 0 || sb_skb < 0 || sb_snb < 0)
        return FP8_ERR_LAYOUT;
    if (!aligned16(a) || lda % 16 != 0 || !aligned16(b) || ldb % 16 != 0 || !aligned16(c) ||
        (ldc * oes) % 16 != 0 || !aligned4(sa) || !aligned4(sb))
        return FP8_ERR_ALIGN;
    if (K / 128 > INT32_MAX / 2 || N > (static_cast<int64_t>(1) << 31)) return FP8_ERR_SHAPE;
    return FP8_OK;
}

fp8_status_t fp8_blockscaled_gemm(const uint8_t* a, int64_t lda, const float* sa,
                                  int64_t sa_stride_m, int64_t sa_stride_kb, const uint8_t* b,
                                  int64_t ldb, int b_kmajor, const float* sb,
                                  int64_t sb_stride_kb, int64_t sb_stride_nb, void* c,
                                  fp8_out_t c_type, int64_t ldc, int64_t M, int64_t N, int64_t K,
                                  fp8_stream_t stream) {
    if (elem_size_out(c_type) == 0) return FP8_ERR_DTYPE;
    if (M < 0 || N < 0 || K < 0 || N % 128 != 0 || K % 128 != 0) return FP8_ERR_SHAPE;
    if (M == 0 || N == 0) return FP8_OK;
    if (!b_kmajor) return FP8_ERR_LAYOUT;
    if (K == 0) return zero_output(c, c_type, ldc, M, N, stream);
    fp8_status_t st = check_gemm_common(a, lda, sa, sa_stride_m, sa_stride_kb, b, ldb, sb,
                                        sb_stride_kb, sb_stride_nb, c, c_type, ldc, N, K);
    if (st != FP8_OK) return st;
    GemmParams out{};
    out.c = c; out.ldc = ldc;
    return dense_gemm<false>(a, lda, sa, sa_stride_m, sa_stride_kb, b, ldb, sb, sb_stride_kb,
                             sb_stride_nb, out, c_type, M, N, K, stream);
}

fp8_status_t fp8_blockscaled_gemm_quant(const uint8_t* a, int64_t lda, const float* sa,
                                        int64_t sa_stride_m, int64_t sa_stride_kb,
                                        const uint8_t* b, int64_t ldb, const float* sb,
                                        int64_t sb_stride_kb, int64_t sb_stride_nb, uint8_t* qc,
                                        int64_t ldqc, float* sc, int64_t sc_stride_m,
                                        int64_t sc_stride_nb, void* c, int64_t ldc, int64_t M,
                                        int64_t N, int64_t K, fp8_stream_t stream) {
    if (M < 0 || N < 0 || K < 0 || N % 128 != 0 || K % 128 != 0) return FP8_ERR_SHAPE;
    if (M == 0 || N == 0) return FP8_OK;
    if (K == 0) return FP8_ERR_SHAPE;
    if (!qc || !sc) return FP8_ERR_NULL;
    if (ldqc < N || sc_stride_m < 0 || sc_stride_nb < 0 || (c && ldc < N)) return FP8_ERR_LAYOUT;
    if (!aligned16(qc) || ldqc % 16 != 0 || !aligned4(sc) ||
        (c && (!aligned16(c) || (ldc * 2) % 16 != 0)))
        return FP8_ERR_ALIGN;
    // The operand checks of the plain GEMM (a stand-in for c when c is null).
    fp8_status_t st = check_gemm_common(a, lda, sa, sa_stride_m, sa_stride_kb, b, ldb, sb,
                                        sb_stride_kb, sb_stride_nb, c ? c : static_cast<void*>(qc),
                                        FP8_OUT_BF16, c ? ldc : N, N, K);
    if (st != FP8_OK) return st;
    GemmParams out{};
    out.c = c; out.ldc = ldc;
    out.qc = qc; out.ldqc = ldqc;
    out.sc = sc; out.sc_sm = sc_stride_m; out.sc_snb = sc_stride_nb;
    return dense_gemm<true>(a, lda, sa, sa_stride_m, sa_stride_kb, b, ldb, sb, sb_stride_kb,
                            sb_stride_nb, out, FP8_OUT_BF16, M, N, K, stream);
}

fp8_status_t fp8_quantize_act_128x1(const void* x, fp8_in_t x_type, int64_t M, int64_t K,
                                    int64_t ldx, uint8_t* qt, int64_t ldq, float* st,
                                    int64_t st_stride_k, int64_t st_stride_mb,
                                    fp8_stream_t stream) {
    const int es = elem_size_in(x_type);
    if (es == 0) return FP8_ERR_DTYPE;
    if (M < 0 || K < 0 || M % 128 != 0 || K % 128 != 0) return FP8_ERR_SHAPE;
    if (M == 0 || K == 0) return FP8_OK;
    if (x_type != FP8_IN_BF16) return FP8_ERR_DTYPE;
    if (!x || !qt || !st) return FP8_ERR_NULL;
    if (ldx < K || ldq < M || st_stride_k < 0 || st_stride_mb < 0) return FP8_ERR_LAYOUT;
    if (!aligned16(x) || (ldx * es) % 16 != 0 || !aligned16(qt) || ldq % 16 != 0 || !aligned4(st))
        return FP8_ERR_ALIGN;
    if (M > INT32_MAX || K > INT32_MAX) return FP8_ERR_SHAPE;
    int dev, sms;
    fp8_status_t s = current_device(&dev, &sms);
    if (s != FP8_OK) return s;
    // Codes that can leave as 32-byte stores: column pairs per thread.
    if (aligned32(qt) && ldq % 32 == 0)
        return launch_quant_weight_rows(x, M, K, ldx, qt, kQwColTiles, ldq, st, st_stride_mb,
                                        st_stride_k, sms, stream);
    QsParams p{};
    p.rows = M; p.cols = K;
    p.nbr = M / 128; p.nbc = K / 128;
    p.q = qt; p.ldq = ldq;
    p.s = st; p.s_stride_r = st_stride_k; p.s_stride_c = st_stride_mb;
    return launch_quant_stream(x, x_type, ldx, p, kQuantActT, sms, stream);
}

fp8_status_t fp8_blockscaled_gemm_colscale(const uint8_t* a, int64_t lda, const float* sa,
                                           int64_t sa_stride_m, int64_t sa_stride_kb,
                                           const uint8_t* b, int64_t ldb, const float* sb,
                                           int64_t sb_stride_kb, void* c, fp8_out_t c_type,
                                           int64_t ldc, int64_t M, int64_t N, int64_t K,
                                           fp8_stream_t stream) {
    if (elem_size_out(c_type) == 0) return FP8_ERR_DTYPE;
    if (M < 0 || N < 0 || K < 0 || N % 128 != 0 || K % 128 != 0) return FP8_ERR_SHAPE;
    if (M == 0 || N == 0) return FP8_OK;
    if (K == 0) return zero_output(c, c_type, ldc, M, N, stream);
    fp8_status_t st = check_gemm_common(a, lda, sa, sa_stride_m, sa_stride_kb, b, ldb, sb,
                                        sb_stride_kb, 1, c, c_type, ldc, N, K);
    if (st != FP8_OK) return st;
    // Each epilogue warp copies its 128 column scales of a chunk as 16-byte
    // pieces.  The row stride matters only when there is more than one chunk.
    const bool multi_chunk = K > 128;
    if (multi_chunk && sb_stride_kb < N) return FP8_ERR_LAYOUT;
    if (!aligned16(sb) || (multi_chunk && sb_stride_kb % 4 != 0)) return FP8_ERR_ALIGN;
    GemmParams out{};
    out.c = c; out.ldc = ldc;
    return dense_gemm<false, true>(a, lda, sa, sa_stride_m, sa_stride_kb, b, ldb, sb, sb_stride_kb,
                                   1, out, c_type, M, N, K, stream);
}

fp8_status_t fp8_grouped_gemm(const uint8_t* a, int64_t lda, const float* sa,
                              int64_t sa_stride_m, int64_t sa_stride_kb, const uint8_t* b,
                              int64_t ldb, const float* sb, int64_t sb_stride_g,
                              int64_t sb_stride_kb, int64_t sb_stride_nb, void* c,
                              fp8_out_t c_type, int64_t ldc, const int32_t* offsets, int G,
                              int64_t total_M, int64_t N, int64_t K, fp8_stream_t stream) {
    if (elem_size_out(c_type) == 0) return FP8_ERR_DTYPE;
    if (G < 1 || G > kMaxGroups || total_M < 0 || N < 0 || K < 0 || N % 128 != 0 || K % 128 != 0)
        return FP8_ERR_SHAPE;
    if (total_M == 0 || N == 0) return FP8_OK;
    if (K == 0) return zero_output(c, c_type, ldc, total_M, N, stream);
    if (!offsets) return FP8_ERR_NULL;
    if (!aligned4(offsets)) return FP8_ERR_ALIGN;
    if (sb_stride_g < 0) return FP8_ERR_LAYOUT;
    fp8_status_t st = check_gemm_common(a, lda, sa, sa_stride_m, sa_stride_kb, b, ldb, sb,
                                        sb_stride_kb, sb_stride_nb, c, c_type, ldc, N, K);
    if (st != FP8_OK) return st;
    const int64_t num_nt = (N + kBN - 1) / kBN;
    const bool use_pair = K >= kGroupedPairMinK;
    // Pair tiles: sum over groups of at most ceil(rows_g / 256); the one-CTA
    // launch: ceil(rows_g / 128) alone, or at most one tile per group after
    // the pair launch.
    const int64_t max_mt = use_pair ? total_M / kPairBM + G : total_M / kBM + G;
    if (total_M > INT32_MAX || max_mt * num_nt > INT32_MAX ||
        static_cast<int64_t>(G) * N > INT32_MAX)
        return FP8_ERR_SHAPE;
    int dev, sms;
    st = current_device(&dev, &sms);
    if (st != FP8_OK) return st;

    CUtensorMap tmA, tmB;
    const uint64_t kcols = static_cast<uint64_t>(K);
    const uint64_t b_rows = static_cast<uint64_t>(G) * static_cast<uint64_t>(N);
    if (!make_operand_map(&tmA, a, static_cast<uint64_t>(total_M), kcols, static_cast<uint64_t>(lda), kBM) ||
        !make_operand_map(&tmB, b, b_rows, kcols, static_cast<uint64_t>(ldb), kBN))
        return FP8_ERR_CUDA;

    GemmParams p{};
    p.sa = sa; p.sa_sm = sa_stride_m; p.sa_skb = sa_stride_kb;
    p.sb = sb; p.sb_sg = sb_stride_g; p.sb_skb = sb_stride_kb; p.sb_snb = sb_stride_nb;
    p.c = c; p.ldc = ldc; p.M = total_M; p.N = N;
    p.c_v8 = (aligned32(c) && (ldc * elem_size_out(c_type)) % 32 == 0) ? 1 : 0;
    p.nkb = static_cast<int>(K / 128);
    p.num_mt = 0;
    p.num_nt = static_cast<int>(num_nt);
    p.band_m = 1;
    p.band_n = 0;
    p.offsets = offsets; p.G = G;
    p.grp_split = kGrpAll;
    if (use_pair) {
        // Whole 256-row blocks (and remainders over 128 rows) on CTA pairs,
        // then each group's remainder of 1-128 rows as one 128-row tile.
        CUtensorMap tmB_pair;   // each CTA of a pair loads 128 rows of B
        if (!make_operand_map(&tmB_pair, b, b_rows, kcols, static_cast<uint64_t>(ldb), 128))
            return FP8_ERR_CUDA;
        p.grp_split = kGrpPairPart;
        st = launch_pair_gemm<true>(tmA, tmB_pair, p,
                                    grid_for(max_mt * num_nt, g_dev[dev].max_pairs, 1), c_type,
                                    stream);
        if (st != FP8_OK) return st;
        p.grp_split = kGrpTailPart;
    }
    const int64_t tail_tiles = use_pair ? static_cast<int64_t>(G) * num_nt : max_mt * num_nt;
    const int64_t grid = grid_for(tail_tiles, sms, 1);
    if (c_type == FP8_OUT_BF16)
        blockscaled_gemm_kernel<true, true>
            <<<static_cast<unsigned>(grid), kGemmThreads, kGemmSmemBytes, stream>>>(tmA, tmB, p);
    else
        blockscaled_gemm_kernel<true, false>
            <<<static_cast<unsigned>(grid), kGemmThreads, kGemmSmemBytes, stream>>>(tmA, tmB, p);
    return launch_status();
}

fp8_status_t fp8_set_wait_limit(int64_t cycles) {
    int dev, sms;
    fp8_status_t st = current_device(&dev, &sms);
    if (st != FP8_OK) return st;
    if (cycles < 0) return FP8_ERR_SHAPE;
    const long long v = cycles == 0 ? kWaitLimitCycles : static_cast<long long>(cycles);
    // Synchronous copy: no kernel of this device runs with a half-written limit.
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpyToSymbol(g_wait_limit_cycles, &v, sizeof v) != cudaSuccess) {
        cudaGetLastError();
        return FP8_ERR_CUDA;
    }
    return FP8_OK;
}

fp8_status_t fp8_get_device_error(fp8_stream_t stream, fp8_status_t* code) {
    if (!code) return FP8_ERR_NULL;
    int dev, sms;
    fp8_status_t st = current_device(&dev, &sms);
    if (st != FP8_OK) return st;
    if (cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaGetLastError();
        return FP8_ERR_CUDA;
    }
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof v) != cudaSuccess ||
        cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero) != cudaSuccess) {
        cudaGetLastError();
        return FP8_ERR_CUDA;
    }
    *code = static_cast<fp8_status_t>(v);
    return FP8_OK;
}

}  // extern "C"
