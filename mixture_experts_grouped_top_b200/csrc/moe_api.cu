// Host side of the C ABI declared in include/moe_grouped.h: argument validation,
// tensor-map construction, launch configuration and the device error word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "moe_grouped.h"
#include "grouped_gemm_kgroup_pair_sm100.cuh"
#include "grouped_gemm_mxf8_kgroup_pair_sm100.cuh"
#include "grouped_gemm_mxf8_pair_sm100.cuh"
#include "grouped_gemm_mxf8_sm100.cuh"
#include "grouped_gemm_pair_sm100.cuh"
#include "grouped_gemm_sm100.cuh"
#include "token_kernels.cuh"

using namespace moe;

namespace {

std::atomic<uint64_t> g_launches{0};

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline int launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    fprintf(stderr, "moe_grouped: launch failed: %s\n", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

inline void count_launch(int n = 1) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

struct DeviceProps {
  int sm_count = 0;
};

DeviceProps& device_props() {
  static DeviceProps props[64];
  static std::once_flag flags[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  std::call_once(flags[dev], [dev]() {
    cudaDeviceGetAttribute(&props[dev].sm_count, cudaDevAttrMultiProcessorCount, dev);
    if (props[dev].sm_count <= 0) props[dev].sm_count = 148;
  });
  return props[dev];
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, []() {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D tiled tensor map (128-byte swizzle unless told otherwise): dims {d0 (contiguous),
// d1, d2}, byte strides of d1 and d2, box {box0, box1, 1}.
int make_tmap(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2,
              uint64_t stride1, uint64_t stride2, uint32_t box0, uint32_t box1,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return MOE_ERR_CUDA;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (stride1 & 15) || (stride2 & 15)) return MOE_ERR_INVALID_ARG;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1, stride2};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fprintf(stderr, "moe_grouped: cuTensorMapEncodeTiled failed (%d)\n", (int)r);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// Stacked matrices [batch, rows, cols] (row-major, elem-byte elements, cols * elem a
// multiple of 128) viewed as 128-byte column chunks: dims {128 / elem, rows, chunks,
// batch}, box {128 / elem, box_rows, box_chunks, 1}. One box lands as box_chunks
// 128-byte-swizzled tiles of box_rows rows back to back ([chunk][row]): the operand layout
// of the CTA-pair kernels (128 rows x 2 chunks) and of the MN-major weight-gradient
// operands (64 k rows x 2 or 4 column chunks).
int tmap_chunks(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t batch, uint64_t rows, uint64_t cols,
                uint32_t elem, uint32_t box_rows = 128, uint32_t box_chunks = 2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return MOE_ERR_CUDA;
  const uint64_t row_bytes = cols * elem;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || (row_bytes % 128)) return MOE_ERR_INVALID_ARG;
  cuuint64_t dims[4] = {128 / elem, rows, row_bytes / 128, batch};
  cuuint64_t strides[3] = {row_bytes, 128, rows * row_bytes};
  cuuint32_t box[4] = {128 / elem, box_rows, box_chunks, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(m, dt, 4, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fprintf(stderr, "moe_grouped: cuTensorMapEncodeTiled (chunked) failed (%d)\n", (int)r);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// CTA-pair kernels: launch as many 2-CTA clusters as can be resident at once (a
// persistent grid larger than that would leave some pairs waiting for others to finish).
// th: the saved h for the SwiGLU backward (any map otherwise: unused).
template <bool B_MN, int EPI>
int launch_gemm_pair(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p, cudaStream_t st,
                     const CUtensorMap* th = nullptr) {
  auto kern = grouped_gemm_bf16_pair_kernel<B_MN, EPI>;
  constexpr int kSmem = g2::smem_bytes(EPI);
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  static int pairs = 0;
  std::call_once(once, [&]() {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (attr_err != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(device_props().sm_count, 1, 1);
    cfg.blockDim = dim3(g2::kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmem;
    cfg.attrs = nullptr;   // the kernel declares its 2-CTA cluster at compile time
    cfg.numAttrs = 0;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) n = device_props().sm_count / 2;
    pairs = std::min(n, device_props().sm_count / 2);
    cudaGetLastError();
  });
  if (attr_err != cudaSuccess) return MOE_ERR_CUDA;
  GemmParams q = p;
  CUtensorMap to = ta;
  if (EPI == EPI_STORE && p.out && p.M > 0 && p.N > 0 && !p.out_f32 && !p.row_token) {
    // bf16 output [M rows, N] as the epilogue's TMA store target: {N, M, 1}, boxes {32, 32}
    if (int rc = make_tmap(&to, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.out, p.N, p.M, 1, (uint64_t)p.ldo * 2,
                           (uint64_t)p.ldo * 2 * p.M, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
      return rc;
    q.tma_out = 1;
  }
  CUtensorMap ty = ta;
  if (EPI == EPI_DSWIGLU) {
    // dh [R, 2F] bf16 as the epilogue's TMA store target: {2F, R, 1}, boxes {32, 32}
    if (p.M == 0) return MOE_OK;
    if (int rc = make_tmap(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.out2, 2 * (uint64_t)p.F, p.M, 1,
                           (uint64_t)p.ldo2 * 2, (uint64_t)p.ldo2 * 2 * p.M, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
      return rc;
  }
  kern<<<2 * pairs, g2::kThreads, kSmem, st>>>(ta, tb, th ? *th : to, ty, q);
  count_launch();
  return launch_status();
}

// BF16 weight-gradient GEMMs on CTA pairs: as many 2-CTA clusters as can be resident.
int launch_wgrad_pair(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p, cudaStream_t st) {
  // dW [E, M, N] bf16 as the epilogue's TMA store target: {N, M, E}, boxes {32, 32}
  CUtensorMap to;
  if (int rc = make_tmap(&to, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.out, p.N, p.M, p.E, (uint64_t)p.ldo * 2,
                         (uint64_t)p.out_batch * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return rc;
  auto kern = grouped_wgrad_bf16_pair_kernel;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  static int pairs = 0;
  std::call_once(once, [&]() {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kp::kSmemBytes);
    if (attr_err != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(device_props().sm_count, 1, 1);
    cfg.blockDim = dim3(kp::kThreads, 1, 1);
    cfg.dynamicSmemBytes = kp::kSmemBytes;
    cfg.attrs = nullptr;
    cfg.numAttrs = 0;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) n = device_props().sm_count / 2;
    pairs = std::min(n, device_props().sm_count / 2);
    cudaGetLastError();
  });
  if (attr_err != cudaSuccess) return MOE_ERR_CUDA;
  kern<<<2 * pairs, kp::kThreads, kp::kSmemBytes, st>>>(ta, tb, to, p);
  count_launch();
  return launch_status();
}

// MMA scale atoms [groups, kb4 atoms of 512 bytes] as a TMA source: uint32 tensor
// {128 words, kb4, groups}, boxes of mx2::kSfKb consecutive atoms of one group (unswizzled).
int tmap_atoms(CUtensorMap* m, const void* atoms, uint64_t groups, uint64_t kb4) {
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, atoms, 128, kb4, groups, 512, kb4 * 512, 128, mx2::kSfKb,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
}

// MXFP8 CTA-pair kernels: as many 2-CTA clusters as can be resident at once.
// th: the saved h for the SwiGLU backward (any map otherwise: unused).
template <int EPI>
int launch_gemm_mx_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsa, const CUtensorMap& tsb,
                        const MxGemmParams& p, cudaStream_t st, const CUtensorMap* th = nullptr) {
  auto kern = grouped_gemm_mxf8_pair_kernel<EPI>;
  constexpr int kSmem = mx2::smem_bytes(EPI);
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  static int pairs = 0;
  std::call_once(once, [&]() {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (attr_err != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(device_props().sm_count, 1, 1);
    cfg.blockDim = dim3(mx2::kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmem;
    cfg.attrs = nullptr;
    cfg.numAttrs = 0;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) n = device_props().sm_count / 2;
    pairs = std::min(n, device_props().sm_count / 2);
    cudaGetLastError();
  });
  if (attr_err != cudaSuccess) return MOE_ERR_CUDA;
  CUtensorMap tdc = ta, tdr = ta;
  if (EPI == MXEPI_DSWIGLU) {
    // dh's code arrays [R, 2F] as the epilogue's TMA store targets: {2F, R, 1}, boxes {32, 32}
    const uint64_t F2 = 2 * (uint64_t)p.g.F, R = (uint64_t)p.g.M;
    if (R == 0) return MOE_OK;
    int rc;
    if ((rc = make_tmap(&tdc, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.dh_cols, F2, R, 1, F2, F2 * R, 32, 32,
                        CU_TENSOR_MAP_SWIZZLE_32B)) ||
        (rc = make_tmap(&tdr, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.dh_rows, F2, R, 1, F2, F2 * R, 32, 32,
                        CU_TENSOR_MAP_SWIZZLE_32B)))
      return rc;
  }
  kern<<<2 * pairs, mx2::kThreads, kSmem, st>>>(ta, tb, tsa, tsb, th ? *th : ta, tdc, tdr, p);
  count_launch();
  return launch_status();
}

// Grouped scale atoms (K-grouped operands: n_atoms of 512 bytes) as a TMA source: uint32
// tensor {128 words, n_atoms, 1}, boxes of mkp::kSfKg consecutive atoms (unswizzled).
int tmap_atoms_flat(CUtensorMap* m, const void* atoms, uint64_t n_atoms) {
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, atoms, 128, n_atoms, 1, 512, n_atoms * 512, 128, mkp::kSfKg,
                   CU_TENSOR_MAP_SWIZZLE_NONE);
}

// MXFP8 weight-gradient GEMM dW[e] = A_e^T B_e on CTA pairs. A codes [R, M], B codes
// [R, N] (MN-major), their grouped atoms (a_atoms / b_atoms hold at least a_n / b_n atoms).
int launch_wgrad_mx_pair(const uint8_t* a, const uint8_t* a_atoms, uint64_t a_n, const uint8_t* b,
                         const uint8_t* b_atoms, uint64_t b_n, int R, const MxGemmParams& p, cudaStream_t st) {
  auto kern = grouped_wgrad_mxf8_pair_kernel;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  static int pairs = 0;
  std::call_once(once, [&]() {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, mkp::kSmemBytes);
    if (attr_err != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(device_props().sm_count, 1, 1);
    cfg.blockDim = dim3(mkp::kThreads, 1, 1);
    cfg.dynamicSmemBytes = mkp::kSmemBytes;
    cfg.attrs = nullptr;
    cfg.numAttrs = 0;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) n = device_props().sm_count / 2;
    pairs = std::min(n, device_props().sm_count / 2);
    cudaGetLastError();
  });
  if (attr_err != cudaSuccess) return MOE_ERR_CUDA;
  if ((p.g.M % 128) || (p.g.N % 128)) return MOE_ERR_UNSUPPORTED;
  CUtensorMap ta, tb, tsa, tsb;
  int rc;
  if ((rc = make_tmap(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a, p.g.M, R, 1, p.g.M, (uint64_t)R * p.g.M, 128,
                      mkp::BK)))
    return rc;
  if ((rc = make_tmap(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, b, p.g.N, R, 1, p.g.N, (uint64_t)R * p.g.N, 128,
                      mkp::BK)))
    return rc;
  if ((rc = tmap_atoms_flat(&tsa, a_atoms, a_n))) return rc;
  if ((rc = tmap_atoms_flat(&tsb, b_atoms, b_n))) return rc;
  kern<<<2 * pairs, mkp::kThreads, mkp::kSmemBytes, st>>>(ta, tb, tsa, tsb, p);
  count_launch();
  return launch_status();
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int quant_rows_launch(const void* in, long long rows, int cols, int mma, uint8_t* codes, uint8_t* scales,
                      cudaStream_t st) {
  const long long nvec = rows * cols / 8;
  const int grid = (int)std::min<long long>((nvec + 255) / 256, (long long)device_props().sm_count * 16);
  quant_rows_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(in), nvec, cols, mma, codes, scales);
  count_launch();
  return launch_status();
}

int quant_cols_grouped_launch(const void* in, int R, int C, const int32_t* split_sizes, int E, uint8_t* codes,
                              uint8_t* atoms, cudaStream_t st) {
  const int blocks32 = R / 32 + E;   // upper bound of sum(ceil(n_e / 32))
  const int ytiles = (C + 511) / 512;   // 256 threads x 2 columns
  dim3 grid(std::min(blocks32, std::max(1, device_props().sm_count * 24 / ytiles)), ytiles);
  quant_cols_grouped_kernel<<<grid, 256, 3 * (E + 1) * sizeof(int32_t), st>>>(
      reinterpret_cast<const __nv_bfloat16*>(in), C, split_sizes, E, codes, atoms);
  count_launch();
  return launch_status();
}

int scales_to_atoms_launch(const uint8_t* plain, const int32_t* split_sizes, int E, int R, int K, uint8_t* atoms,
                           cudaStream_t st) {
  const long long words = ((long long)R / 128 + E) * (K / 128) * 128;
  const int grid = (int)std::min<long long>((words + 255) / 256, (long long)device_props().sm_count * 8);
  scales_to_atoms_kernel<<<grid, 256, 2 * (E + 1) * sizeof(int32_t), st>>>(
      plain, split_sizes, E, K / 32, (long long)R / 128 + E, reinterpret_cast<uint32_t*>(atoms));
  count_launch();
  return launch_status();
}

// Bytes of MMA scale atoms for R expert-contiguous rows of K values: at most R/128 + E
// row groups (one partial group per expert), K/128 atoms of 512 bytes each.
size_t mma_atoms_bytes(int E, int R, int K) {
  return align_up(((size_t)R / 128 + (size_t)E) * (size_t)(K / 128) * 512, 256);
}

// Launch helpers used by the MXFP8 backward (all asynchronous on `st`).
int quant_rows_launch(const void* in, long long rows, int cols, int mma, uint8_t* codes, uint8_t* scales,
                      cudaStream_t st);
int quant_cols_grouped_launch(const void* in, int R, int C, const int32_t* split_sizes, int E, uint8_t* codes,
                              uint8_t* atoms, cudaStream_t st);
int scales_to_atoms_launch(const uint8_t* plain, const int32_t* split_sizes, int E, int R, int K, uint8_t* atoms,
                           cudaStream_t st);

// One-shot stall armed by moe_test_stall_gemm: the wait budget of the stalled launch (0 =
// none armed) and how many grouped GEMM launches to let through before it.
std::atomic<uint64_t> g_stall_ns{0};
std::atomic<int> g_stall_skip{0};

GemmParams base_params(const int32_t* split_sizes, int E) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.E = E;
  p.split_sizes = split_sizes;
  p.timeout_ns = gg::kTimeoutNs;
  const uint64_t stall = g_stall_ns.load();
  if (stall && g_stall_skip.fetch_sub(1) == 0) {
    g_stall_ns.store(0);
    p.timeout_ns = stall;
    p.stall_loads = 1;
  }
  return p;
}

// ---------------------------------------------------------------- per-tensor FP8
int fp8_amax_launch(const void* in, int batch, long long n, unsigned int* amax, cudaStream_t st) {
  if (cudaMemsetAsync(amax, 0, (size_t)batch * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
  const long long n8 = n / 8;
  if (n8 == 0) return MOE_OK;
  const int gx = (int)std::max<long long>(1, std::min<long long>((n8 + 255) / 256,
                                                                 (long long)device_props().sm_count * 8 / batch + 1));
  amax_bf16_kernel<<<dim3(gx, batch), 256, 0, st>>>(reinterpret_cast<const uint4*>(in), n8, amax);
  count_launch();
  return launch_status();
}

int fp8_scale_launch(const unsigned int* amax, int batch, int e5m2, float* scale, cudaStream_t st) {
  fp8_scale_kernel<<<(batch + 255) / 256, 256, 0, st>>>(amax, batch, e5m2, scale);
  count_launch();
  return launch_status();
}

int fp8_cast_launch(const void* in, int batch, long long n, const float* scale, int e5m2, uint8_t* codes,
                    cudaStream_t st) {
  const long long n8 = n / 8;
  if (n8 == 0) return MOE_OK;
  const int gx = (int)std::max<long long>(1, std::min<long long>((n8 + 255) / 256,
                                                                 (long long)device_props().sm_count * 8 / batch + 1));
  fp8_cast_kernel<<<dim3(gx, batch), 256, 0, st>>>(reinterpret_cast<const uint4*>(in), n8, scale, e5m2,
                                                    reinterpret_cast<uint2*>(codes));
  count_launch();
  return launch_status();
}

// amax, scale and codes of `batch` tensors of n bf16 each (codes in the input's layout)
int fp8_quantize_launch(const void* in, int batch, long long n, int e5m2, uint8_t* codes, float* scale,
                        unsigned int* amax, cudaStream_t st) {
  int rc;
  if ((rc = fp8_amax_launch(in, batch, n, amax, st))) return rc;
  if ((rc = fp8_scale_launch(amax, batch, e5m2, scale, st))) return rc;
  return fp8_cast_launch(in, batch, n, scale, e5m2, codes, st);
}

// Block-scale atoms of per-tensor FP8 operands: every scale byte 127 (2^0), enough for
// every A and B operand of the layer's grouped GEMMs.
size_t fp8_unit_atoms_bytes(int E, int R, int H, int F) {
  const size_t a = ((size_t)R / 128 + (size_t)E) * (size_t)(std::max(H, 2 * F) / 128);
  const size_t b = (size_t)E * (size_t)(2 * F / 128) * (size_t)(H / 128);
  return align_up(std::max(a, b) * 512, 256);
}

}  // namespace

extern "C" {

size_t fp8_quantize_workspace_size(int batch) { return batch < 1 ? 0 : align_up((size_t)batch * 4, 256); }

int fp8_quantize(const uint16_t* in, int batch, int rows, int cols, int fmt, int transpose_out, uint8_t* codes,
                 float* scales, void* workspace, size_t workspace_bytes, void* stream) {
  if (batch < 1 || rows < 0 || cols < 0 || (fmt != 0 && fmt != 1)) return MOE_ERR_INVALID_ARG;
  const long long n = (long long)rows * cols;
  if (n == 0) return MOE_OK;
  if (!in || !codes || !scales || !workspace) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < fp8_quantize_workspace_size(batch)) return MOE_ERR_INVALID_ARG;
  if (transpose_out ? ((rows % 32) || (cols % 32)) : (n % 8)) return MOE_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(in) & 15) || (reinterpret_cast<uintptr_t>(codes) & 7)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  unsigned int* amax = reinterpret_cast<unsigned int*>(workspace);
  int rc;
  if ((rc = fp8_amax_launch(in, batch, n, amax, st))) return rc;
  if ((rc = fp8_scale_launch(amax, batch, fmt, scales, st))) return rc;
  if (!transpose_out) return fp8_cast_launch(in, batch, n, scales, fmt, codes, st);
  fp8_cast_transpose_kernel<<<dim3(cols / 32, rows / 32, batch), 256, 0, st>>>(
      reinterpret_cast<const __nv_bfloat16*>(in), rows, cols, scales, fmt, codes);
  count_launch();
  return launch_status();
}

const char* moe_status_string(int s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    default: return "MOE_ERR_UNKNOWN";
  }
}

uint64_t moe_launch_count(void) { return g_launches.load(); }

int moe_test_stall_gemm(int skip, uint64_t timeout_ns) {
  if (skip < 0 || timeout_ns < 100000ull || timeout_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;
  g_stall_skip.store(skip);
  g_stall_ns.store(timeout_ns);
  return MOE_OK;
}

int moe_device_status(void* stream) {
  cudaStream_t st = as_stream(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  int h = 0;
  if (cudaMemcpyFromSymbol(&h, g_device_error, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  if (h) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (h & DEVERR_TIMEOUT) return MOE_ERR_TIMEOUT;
  if (h) return MOE_ERR_DEVICE_CHECK;
  return MOE_OK;
}

int moe_route(const float* logits, int T, int E, int k, int renorm, int32_t* idx, float* prob, void* stream) {
  if (T < 0 || E < 1 || E > kMaxExperts || k < 1 || k > E || k > 32) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!logits || !idx || !prob) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  const int threads = 256, wpb = threads / 32;
  const int grid = std::min((T + wpb - 1) / wpb, device_props().sm_count * 16);
  const int vpl = (E + 31) / 32;
#define MOE_ROUTE_CASE(V) \
  case V: route_topk_kernel<V><<<grid, threads, 0, st>>>(logits, T, E, k, renorm, idx, prob); break;
  switch (vpl <= 1 ? 1 : vpl <= 2 ? 2 : vpl <= 4 ? 4 : vpl <= 8 ? 8 : vpl <= 16 ? 16 : 32) {
    MOE_ROUTE_CASE(1)
    MOE_ROUTE_CASE(2)
    MOE_ROUTE_CASE(4)
    MOE_ROUTE_CASE(8)
    MOE_ROUTE_CASE(16)
    MOE_ROUTE_CASE(32)
  }
#undef MOE_ROUTE_CASE
  count_launch();
  return launch_status();
}

int moe_route_bwd(const float* logits, const int32_t* idx, const float* prob, const float* dprob, int T, int E,
                  int k, int renorm, float* dlogits, void* stream) {
  if (T < 0 || E < 1 || E > kMaxExperts || k < 1 || k > E || k > 32) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!idx || !prob || !dprob || !dlogits || (!renorm && !logits)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  const int threads = 256, wpb = threads / 32;
  const int grid = std::min((T + wpb - 1) / wpb, device_props().sm_count * 16);
  const int vpl = (E + 31) / 32;
#define MOE_ROUTE_BWD_CASE(V)                                                                              \
  case V:                                                                                                  \
    route_bwd_kernel<V><<<grid, threads, 0, st>>>(logits, idx, prob, dprob, T, E, k, renorm, dlogits); \
    break;
  switch (vpl <= 1 ? 1 : vpl <= 2 ? 2 : vpl <= 4 ? 4 : vpl <= 8 ? 8 : vpl <= 16 ? 16 : 32) {
    MOE_ROUTE_BWD_CASE(1)
    MOE_ROUTE_BWD_CASE(2)
    MOE_ROUTE_BWD_CASE(4)
    MOE_ROUTE_BWD_CASE(8)
    MOE_ROUTE_BWD_CASE(16)
    MOE_ROUTE_BWD_CASE(32)
  }
#undef MOE_ROUTE_BWD_CASE
  count_launch();
  return launch_status();
}

namespace {
// counts table of the index build, then (256-byte aligned) the fused path's counter
size_t permute_counts_bytes(size_t R, int E) {
  const size_t nblk = (R + kPermuteChunk - 1) / kPermuteChunk;
  return align_up(std::max<size_t>(nblk, 1) * E * sizeof(int32_t), 256);
}
}  // namespace

size_t moe_permute_workspace_size(int T, int k, int E) {
  if (T < 0 || k < 1 || E < 1) return 0;
  return permute_counts_bytes((size_t)T * k, E) + 256;
}

int moe_permute_rows(const uint16_t* src, const int32_t* row_map, int T, int H, int k, uint16_t* dst, void* stream) {
  if (T < 0 || H < 8 || (H % 8) || k < 1 || k > 32) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!src || !row_map || !dst) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  const int grid = std::min((T + 7) / 8, device_props().sm_count * 8);
  permute_rows_bf16_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(src), T, H / 8, k, row_map,
                                                 reinterpret_cast<uint4*>(dst));
  count_launch();
  return launch_status();
}

size_t moe_permute_rows_mxfp8_workspace_size(int T, int k) {
  if (T < 0 || k < 1) return 0;
  return ((size_t)T * k * 4 + 255) / 256 * 256 + 256;
}

int moe_permute_rows_mxfp8(const uint16_t* src, const int32_t* row_map, int T, int H, int k,
                           const int32_t* split_sizes, int E, uint8_t* rows_codes, uint8_t* rows_atoms,
                           uint8_t* cols_codes, uint8_t* cols_atoms, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (T < 0 || H < 128 || k < 1 || k > 32 || E < 1 || E > kMaxExperts) return MOE_ERR_INVALID_ARG;
  if (H % 128) return MOE_ERR_UNSUPPORTED;
  const long long R = (long long)T * k;
  if (R > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  if ((rows_codes == nullptr) != (rows_atoms == nullptr) || (cols_codes == nullptr) != (cols_atoms == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (R == 0 || (!rows_codes && !cols_codes)) return MOE_OK;
  if (!src || !row_map || !split_sizes || !workspace) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < moe_permute_rows_mxfp8_workspace_size(T, k)) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(rows_codes) |
       reinterpret_cast<uintptr_t>(cols_codes)) & 15)
    return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  int32_t* row_token = reinterpret_cast<int32_t*>(workspace);
  row_token_kernel<<<std::min((int)((R + 255) / 256), device_props().sm_count * 8), 256, 0, st>>>(row_map, (int)R, k,
                                                                                               row_token);
  count_launch();
  int rc;
  if ((rc = launch_status())) return rc;
  const size_t atoms = mma_atoms_bytes(E, (int)R, H);
  if (rows_atoms && cudaMemsetAsync(rows_atoms, 0, atoms, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (cols_atoms && cudaMemsetAsync(cols_atoms, 0, atoms, st) != cudaSuccess) return MOE_ERR_CUDA;
  const int blocks32 = (int)std::min<long long>(R / 32 + E, (long long)device_props().sm_count * 8);
  dim3 grid(blocks32, (H + 255) / 256);
  permute_quant_both_kernel<<<grid, 256, 3 * (E + 1) * sizeof(int32_t), st>>>(
      reinterpret_cast<const __nv_bfloat16*>(src), H, row_token, split_sizes, E, rows_codes, rows_atoms, cols_codes,
      cols_atoms);
  count_launch();
  return launch_status();
}

namespace {
int permute_rows_from_counts(const uint16_t* x, const int32_t* idx, const float* prob, int T, int H, int E, int k,
                             int precision, void* xp, uint8_t* xp_scale, int32_t* row_map, float* probs_perm,
                             const int32_t* counts, cudaStream_t st);
}  // namespace

int moe_permute(const uint16_t* x, const int32_t* idx, const float* prob, int T, int H, int E, int k, int precision,
                void* xp, uint8_t* xp_scale, int32_t* row_map, float* probs_perm, int32_t* split_sizes,
                int32_t* offsets, void* workspace, size_t workspace_bytes, void* stream) {
  if (T < 0 || E < 1 || E > kMaxExperts || k < 1 || k > E || k > 32 || H < 8) return MOE_ERR_INVALID_ARG;
  if (precision != MOE_BF16 && precision != MOE_MXFP8) return MOE_ERR_INVALID_ARG;
  if (precision == MOE_BF16 && (H % 8)) return MOE_ERR_UNSUPPORTED;
  if (precision == MOE_MXFP8 && (H % 32)) return MOE_ERR_UNSUPPORTED;
  if (!split_sizes || !offsets) return MOE_ERR_INVALID_ARG;
  if (probs_perm && !prob) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  const long long R = (long long)T * k;
  if (R > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  if (T > 0 && (!x || !idx || !xp || !row_map || !workspace)) return MOE_ERR_INVALID_ARG;
  if (precision == MOE_MXFP8 && T > 0 && !xp_scale) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < permute_counts_bytes((size_t)R, E)) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(xp)) & 15) return MOE_ERR_INVALID_ARG;
  if (R == 0) {
    // no rows: every expert is empty
    if (cudaMemsetAsync(split_sizes, 0, E * sizeof(int32_t), st) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, (E + 1) * sizeof(int32_t), st) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  const int nblk = (int)((R + kPermuteChunk - 1) / kPermuteChunk);
  int32_t* counts = reinterpret_cast<int32_t*>(workspace);
  permute_hist_kernel<<<nblk, kPermuteThreads, E * sizeof(int32_t), st>>>(idx, (int)R, E, counts);
  const int P = std::max(1, 1024 / E);
  permute_scan_kernel<<<1, 1024, (size_t)(P * E + E) * sizeof(int32_t), st>>>(counts, nblk, E, (int)R, split_sizes,
                                                                                offsets);
  count_launch(2);
  return permute_rows_from_counts(x, idx, prob, T, H, E, k, precision, xp, xp_scale, row_map, probs_perm, counts,
                                  st);
}

namespace {
// Passes 3 and 4 of the permutation: stable ranks (row_map, probs_perm) from the scanned
// counts, then the data movement (with the MXFP8 row quantisation).
int permute_rows_from_counts(const uint16_t* x, const int32_t* idx, const float* prob, int T, int H, int E, int k,
                             int precision, void* xp, uint8_t* xp_scale, int32_t* row_map, float* probs_perm,
                             const int32_t* counts, cudaStream_t st) {
  const long long R = (long long)T * k;
  const int nblk = (int)((R + kPermuteChunk - 1) / kPermuteChunk);
  static std::once_flag once;
  std::call_once(once, []() {
    cudaFuncSetAttribute(permute_rowmap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 8 * kMaxExperts * 4);
  });
  permute_rowmap_kernel<<<nblk, kPermuteThreads, (size_t)(kPermuteThreads / 32) * E * sizeof(int32_t), st>>>(
      idx, prob, (int)R, E, counts, row_map, probs_perm);
  const int grid = std::min((T + 7) / 8, device_props().sm_count * 8);
  if (precision == MOE_BF16) {
    permute_rows_bf16_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(x), T, H / 8, k, row_map,
                                                   reinterpret_cast<uint4*>(xp));
  } else {
    permute_rows_mxfp8_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(x), T, H, k, row_map,
                                                    reinterpret_cast<uint8_t*>(xp), xp_scale);
  }
  count_launch(2);
  return launch_status();
}
}  // namespace

int moe_route_permute(const float* logits, const uint16_t* x, int T, int H, int E, int k, int renorm, int precision,
                      int32_t* idx, float* prob, void* xp, uint8_t* xp_scale, int32_t* row_map, float* probs_perm,
                      int32_t* split_sizes, int32_t* offsets, void* workspace, size_t workspace_bytes,
                      void* stream) {
  if (T < 0 || E < 1 || E > kMaxExperts || k < 1 || k > E || k > 32 || H < 8) return MOE_ERR_INVALID_ARG;
  if (precision != MOE_BF16 && precision != MOE_MXFP8) return MOE_ERR_INVALID_ARG;
  if (precision == MOE_BF16 && (H % 8)) return MOE_ERR_UNSUPPORTED;
  if (precision == MOE_MXFP8 && (H % 32)) return MOE_ERR_UNSUPPORTED;
  if (!split_sizes || !offsets) return MOE_ERR_INVALID_ARG;
  const long long R = (long long)T * k;
  if (R > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  if (T > 0 && (!logits || !x || !idx || !prob || !xp || !row_map || !workspace)) return MOE_ERR_INVALID_ARG;
  if (precision == MOE_MXFP8 && T > 0 && !xp_scale) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < moe_permute_workspace_size(T, k, E)) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(xp)) & 15) return MOE_ERR_INVALID_ARG;
  if (T == 0)
    return moe_permute(x, idx, prob, T, H, E, k, precision, xp, xp_scale, row_map, probs_perm, split_sizes, offsets,
                       workspace, workspace_bytes, stream);
  const int vpl = (E + 31) / 32;
  if ((kPermuteChunk % k) != 0 || vpl > 8) {
    // outside the fused kernel's shapes: the two calls it stands for
    const int rc = moe_route(logits, T, E, k, renorm, idx, prob, stream);
    if (rc != MOE_OK) return rc;
    return moe_permute(x, idx, prob, T, H, E, k, precision, xp, xp_scale, row_map, probs_perm, split_sizes, offsets,
                       workspace, workspace_bytes, stream);
  }
  cudaStream_t st = as_stream(stream);
  const int nblk = (int)((R + kPermuteChunk - 1) / kPermuteChunk);
  int32_t* counts = reinterpret_cast<int32_t*>(workspace);
  unsigned int* done =
      reinterpret_cast<unsigned int*>(reinterpret_cast<uint8_t*>(workspace) + permute_counts_bytes((size_t)R, E));
  if (cudaMemsetAsync(done, 0, sizeof(unsigned int), st) != cudaSuccess) return MOE_ERR_CUDA;
  const int P = std::max(1, 1024 / E);
  const size_t smem = (size_t)std::max(E, (P + 1) * E) * sizeof(int32_t);
#define MOE_ROUTE_INDEX_CASE(C, V, W)                                                                          \
  case C:                                                                                                      \
    route_index_kernel<V, W><<<nblk, 1024, smem, st>>>(logits, T, E, k, renorm, idx, prob, counts, nblk,         \
                                                       split_sizes, offsets, done);                             \
    break;
  // up to 8 or 16 experts: 8 or 16 lanes per token
  switch (E <= 8 ? 0 : E <= 16 ? 1 : vpl <= 1 ? 2 : vpl <= 2 ? 3 : vpl <= 4 ? 4 : 5) {
    MOE_ROUTE_INDEX_CASE(0, 1, 8)
    MOE_ROUTE_INDEX_CASE(1, 1, 16)
    MOE_ROUTE_INDEX_CASE(2, 1, 32)
    MOE_ROUTE_INDEX_CASE(3, 2, 32)
    MOE_ROUTE_INDEX_CASE(4, 4, 32)
    MOE_ROUTE_INDEX_CASE(5, 8, 32)
  }
#undef MOE_ROUTE_INDEX_CASE
  count_launch();
  const int rc = launch_status();
  if (rc != MOE_OK) return rc;
  return permute_rows_from_counts(x, idx, prob, T, H, E, k, precision, xp, xp_scale, row_map, probs_perm, counts, st);
}

size_t moe_permute_capacity_workspace_size(int T, int k, int E) {
  if (T < 0 || k < 1 || E < 1) return 0;
  const size_t R = (size_t)T * k;
  return permute_counts_bytes(R, E) + align_up(R * 4, 256) + 2 * align_up(((size_t)E + 1) * 4, 256);
}

int moe_permute_capacity(const uint16_t* x, const int32_t* idx, const float* prob, int T, int H, int E, int k, int C,
                         int precision, void* xp, uint8_t* xp_scale, int32_t* row_map, float* probs_perm,
                         int32_t* split_sizes, int32_t* offsets, int32_t* kept, void* workspace,
                         size_t workspace_bytes, void* stream) {
  if (T < 0 || E < 1 || E > kMaxExperts || k < 1 || k > E || k > 32 || H < 8 || C < 0) return MOE_ERR_INVALID_ARG;
  if (precision != MOE_BF16 && precision != MOE_MXFP8) return MOE_ERR_INVALID_ARG;
  if (precision == MOE_BF16 && (H % 8)) return MOE_ERR_UNSUPPORTED;
  if (precision == MOE_MXFP8 && (H % 32)) return MOE_ERR_UNSUPPORTED;
  if (probs_perm && !prob) return MOE_ERR_INVALID_ARG;
  const long long R = (long long)T * k, RC = (long long)E * C;
  if (R > 0x7fffffffLL || RC > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  if (!split_sizes || !offsets || (T > 0 && (!x || !idx || !xp || !row_map || !workspace))) return MOE_ERR_INVALID_ARG;
  if (precision == MOE_MXFP8 && T > 0 && !xp_scale) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < moe_permute_capacity_workspace_size(T, k, E)) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(xp)) & 15) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  // the padded rows of every expert hold zeros (their outputs are never combined, and a
  // backward through them contributes nothing to the weight gradients)
  const size_t elem = precision == MOE_BF16 ? 2 : 1;
  if (RC > 0 && cudaMemsetAsync(xp, 0, (size_t)RC * H * elem, st) != cudaSuccess) return MOE_ERR_CUDA;
  if (RC > 0 && precision == MOE_MXFP8 && cudaMemsetAsync(xp_scale, 0, (size_t)RC * (H / 32), st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (RC > 0 && probs_perm && cudaMemsetAsync(probs_perm, 0, (size_t)RC * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
  uint8_t* w = reinterpret_cast<uint8_t*>(workspace);
  int32_t* counts = reinterpret_cast<int32_t*>(w);
  int32_t* row_full = reinterpret_cast<int32_t*>(w + permute_counts_bytes((size_t)R, E));
  int32_t* split_full = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(row_full) + align_up((size_t)R * 4, 256));
  int32_t* off_full =
      reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(split_full) + align_up(((size_t)E + 1) * 4, 256));
  if (R == 0) {
    if (cudaMemsetAsync(split_full, 0, E * sizeof(int32_t), st) != cudaSuccess ||
        cudaMemsetAsync(off_full, 0, (E + 1) * sizeof(int32_t), st) != cudaSuccess)
      return MOE_ERR_CUDA;
  } else {
    // the dropless stable permutation's index (rows only: no data, no probabilities)
    const int nblk = (int)((R + kPermuteChunk - 1) / kPermuteChunk);
    permute_hist_kernel<<<nblk, kPermuteThreads, E * sizeof(int32_t), st>>>(idx, (int)R, E, counts);
    const int P = std::max(1, 1024 / E);
    permute_scan_kernel<<<1, 1024, (size_t)(P * E + E) * sizeof(int32_t), st>>>(counts, nblk, E, (int)R, split_full,
                                                                                  off_full);
    static std::once_flag once;
    std::call_once(once, []() {
      cudaFuncSetAttribute(permute_rowmap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 8 * kMaxExperts * 4);
    });
    permute_rowmap_kernel<<<nblk, kPermuteThreads, (size_t)(kPermuteThreads / 32) * E * sizeof(int32_t), st>>>(
        idx, nullptr, (int)R, E, counts, row_full, nullptr);
    count_launch(3);
  }
  const long long work = std::max<long long>(R, E);
  const int cgrid = (int)std::min<long long>((work + 255) / 256, (long long)device_props().sm_count * 8);
  capacity_rows_kernel<<<cgrid, 256, 0, st>>>(idx, row_full, split_full, off_full, prob, (int)R, E, C, row_map,
                                              probs_perm, split_sizes, offsets, kept);
  count_launch();
  if (R > 0) {
    const int grid = std::min((T + 7) / 8, device_props().sm_count * 8);
    if (precision == MOE_BF16)
      permute_rows_bf16_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(x), T, H / 8, k, row_map,
                                                     reinterpret_cast<uint4*>(xp));
    else
      permute_rows_mxfp8_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(x), T, H, k, row_map,
                                                      reinterpret_cast<uint8_t*>(xp), xp_scale);
    count_launch();
  }
  return launch_status();
}

int moe_unpermute(const uint16_t* yp, const int32_t* row_map, const float* prob, int T, int H, int k, uint16_t* out,
                  void* stream) {
  if (T < 0 || H < 8 || (H % 8) || k < 1 || k > 32) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!yp || !row_map || !out) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(yp) | reinterpret_cast<uintptr_t>(out)) & 15) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  const int grid = std::min((T + 7) / 8, device_props().sm_count * 8);
  unpermute_bf16_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(yp), row_map, prob, T, H / 8, k,
                                              reinterpret_cast<uint4*>(out));
  count_launch();
  return launch_status();
}

int moe_gather_slots(const float* src, const int32_t* row_map, int R, float* dst, void* stream) {
  if (R < 0) return MOE_ERR_INVALID_ARG;
  if (R == 0) return MOE_OK;
  if (!src || !row_map || !dst) return MOE_ERR_INVALID_ARG;
  const int grid = std::min((R + 255) / 256, device_props().sm_count * 4);
  gather_slots_f32_kernel<<<grid, 256, 0, as_stream(stream)>>>(src, row_map, R, dst);
  count_launch();
  return launch_status();
}

int mxfp8_quantize(const uint16_t* in, int batch, int rows, int cols, int axis, int transpose_out,
                   int scale_layout, uint8_t* codes, uint8_t* scales, void* stream) {
  if (batch < 0 || rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
  if (axis != 0 && axis != 1) return MOE_ERR_INVALID_ARG;
  if (axis == 0 && transpose_out) return MOE_ERR_INVALID_ARG;
  if (scale_layout != MOE_SCALES_PLAIN && scale_layout != MOE_SCALES_MMA) return MOE_ERR_INVALID_ARG;
  if (scale_layout == MOE_SCALES_MMA && !((axis == 1 && transpose_out) || (axis == 0 && !transpose_out)))
    return MOE_ERR_INVALID_ARG;
  if (scale_layout == MOE_SCALES_MMA && ((rows % 128) || (cols % 128))) return MOE_ERR_UNSUPPORTED;
  if ((long long)batch * rows * cols == 0) return MOE_OK;
  if (!in || !codes || !scales) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  if (axis == 0) {
    if (cols % 32) return MOE_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(in) & 15) || (reinterpret_cast<uintptr_t>(codes) & 7))
      return MOE_ERR_INVALID_ARG;
    const long long nvec = (long long)batch * rows * cols / 8;
    const long long want = (nvec + 255) / 256;
    const int grid = (int)std::min<long long>(want, (long long)device_props().sm_count * 16);
    quant_rows_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(in), nvec, cols,
                                            scale_layout == MOE_SCALES_MMA, codes, scales);
  } else {
    if (rows % 32) return MOE_ERR_UNSUPPORTED;
    if (transpose_out && (reinterpret_cast<uintptr_t>(codes) & 15)) return MOE_ERR_INVALID_ARG;
    if (batch > 65535 || rows / 32 > 65535) return MOE_ERR_UNSUPPORTED;
    dim3 grid((cols + 255) / 256, rows / 32, batch);
    quant_cols_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(in), rows, cols, transpose_out,
                                            scale_layout == MOE_SCALES_MMA, codes, scales);
  }
  count_launch();
  return launch_status();
}

int mxfp8_quantize_weights(const uint16_t* w, int batch, int rows, int cols, uint8_t* codes_t, uint8_t* atoms_t,
                           uint8_t* codes_r, uint8_t* atoms_r, void* stream) {
  if (batch < 0 || rows < 0 || cols < 0) return MOE_ERR_INVALID_ARG;
  if ((rows % 128) || (cols % 128)) return MOE_ERR_UNSUPPORTED;
  if ((long long)batch * rows * cols == 0) return MOE_OK;
  if (!w || !codes_t || !atoms_t || !codes_r || !atoms_r) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(codes_t) | reinterpret_cast<uintptr_t>(codes_r)) &
      15)
    return MOE_ERR_INVALID_ARG;
  if (batch > 65535) return MOE_ERR_UNSUPPORTED;
  cudaStream_t st = as_stream(stream);
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, []() {
    attr_err = cudaFuncSetAttribute(quant_weights_both_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    qw::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return MOE_ERR_CUDA;
  if (rows / 128 > 65535) return MOE_ERR_UNSUPPORTED;
  dim3 grid(cols / 128, rows / 128, batch);
  quant_weights_both_kernel<<<grid, 256, qw::kSmemBytes, st>>>(reinterpret_cast<const __nv_bfloat16*>(w), rows, cols,
                                                               codes_t, atoms_t, codes_r, atoms_r);
  count_launch();
  return launch_status();
}

size_t grouped_mlp_workspace_size(int E, int R, int H, int F, int precision, int training) {
  (void)E;
  (void)H;
  if (R < 0 || F < 0) return 0;
  if (precision == MOE_FP8) {
    // unit block scales, the max word, a in bf16; a's codes and scale unless in `saved`
    size_t b = fp8_unit_atoms_bytes(E, R, H, F) + 256 + align_up((size_t)R * F * 2, 256);
    if (!training) b += align_up((size_t)R * F, 256) + 256;
    return b + 256;
  }
  if (training && precision != MOE_MXFP8) return 256;  // `a` lives in the saved buffer
  if (precision == MOE_MXFP8) {
    // xp scale atoms, plus `a` codes and scale atoms unless they live in the saved buffer
    const size_t xa = mma_atoms_bytes(E, R, H);
    if (training) return xa + 256;
    return xa + align_up((size_t)R * F, 256) + mma_atoms_bytes(E, R, F) + 256;
  }
  return align_up((size_t)R * F * 2, 256) + 256;
}

size_t grouped_mlp_saved_offset(int E, int R, int H, int F, int precision, int part) {
  if (R < 0 || F < 0 || E < 1 || part < 0) return (size_t)-1;
  const size_t h = align_up((size_t)R * 2 * F * 2, 256), a = align_up((size_t)R * F, 256);
  if (part == 0) return 0;
  if (precision == MOE_MXFP8) {
    const size_t at = mma_atoms_bytes(E, R, F);
    switch (part) {
      case 1: return h;                  // a codes along F (fc2's A)
      case 2: return h + a;              // their scale atoms (tile groups)
      case 3: return h + a + at;         // a codes along the expert's rows (fc2 wgrad's A)
      case 4: return h + 2 * a + at;     // their atoms (grouped)
      default: return (size_t)-1;
    }
  }
  if (precision == MOE_FP8) {
    if (part == 1) return h;             // a E4M3 codes
    if (part == 2) return h + a;         // a's fp32 scale
    return (size_t)-1;
  }
  return part == 1 ? h : (size_t)-1;     // BF16: a bf16
}

size_t grouped_mlp_saved_size(int E, int R, int H, int F, int precision) {
  (void)E;
  (void)H;
  if (R < 0 || F < 0) return 0;
  if (precision == MOE_FP8)   // h bf16, a's E4M3 codes, a's scale
    return align_up((size_t)R * 2 * F * 2, 256) + align_up((size_t)R * F, 256) + 256;
  if (precision == MOE_MXFP8)   // h; a along F (fc2) and along the expert's rows (fc2 wgrad)
    return align_up((size_t)R * 2 * F * 2, 256) + 2 * (align_up((size_t)R * F, 256) + mma_atoms_bytes(E, R, F));
  return align_up((size_t)R * 2 * F * 2, 256) + align_up((size_t)R * F * 2, 256);
}

}  // extern "C"

namespace {

int grouped_mlp_fwd_mxfp8(const void* xp, const uint8_t* xp_scale, const int32_t* split_sizes, int E, int R, int H,
                          int F, const void* w1, const uint8_t* w1_scale, const void* w2, const uint8_t* w2_scale,
                          const float* probs_perm, void* yp, int out_f32, void* saved, void* ws, cudaStream_t st,
                          const int32_t* row_token, float* out32) {
  if ((H % 128) || (F % 128)) return MOE_ERR_UNSUPPORTED;
  if (!xp_scale || !w1_scale || !w2_scale) return MOE_ERR_INVALID_ARG;
  // workspace: xp scale atoms [, a codes, a scale atoms]; training keeps a in `saved`
  uint8_t* xp_atoms = reinterpret_cast<uint8_t*>(ws);
  uint8_t* a_codes = xp_atoms + mma_atoms_bytes(E, R, H);
  uint16_t* h_buf = nullptr;
  if (saved) {
    h_buf = reinterpret_cast<uint16_t*>(saved);
    a_codes = reinterpret_cast<uint8_t*>(saved) + align_up((size_t)R * 2 * F * 2, 256);
  }
  uint8_t* a_atoms = a_codes + align_up((size_t)R * F, 256);
  CUtensorMap ta, tb;
  int rc;
  if ((rc = scales_to_atoms_launch(xp_scale, split_sizes, E, R, H, xp_atoms, st))) return rc;
  // training: the fc1 epilogue also quantises a along the expert's rows (fc2 wgrad operand)
  uint8_t* a_cols = saved ? a_atoms + mma_atoms_bytes(E, R, F) : nullptr;
  uint8_t* a_cols_atoms = saved ? a_cols + align_up((size_t)R * F, 256) : nullptr;
  // fc1: A = xp codes [R, H], B = w1 codes [E, 2F, H] (both K-major)
  if ((rc = tmap_chunks(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, xp, 1, R, H, 1, 128, mx2::kChunks))) return rc;
  if ((rc = tmap_chunks(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w1, E, 2 * F, H, 1, 128, mx2::kChunks))) return rc;
  MxGemmParams p1{};
  p1.g = base_params(split_sizes, E);
  p1.g.M = R;
  p1.g.N = F;
  p1.g.K = H;
  p1.g.out = a_codes;
  p1.g.ldo = F;
  p1.g.out2 = h_buf;
  p1.g.ldo2 = 2 * F;
  p1.g.probs = probs_perm;
  p1.g.F = F;
  p1.a_atoms = xp_atoms;
  p1.b_atoms = w1_scale;
  p1.b_rows = 2 * F;
  p1.out_atoms = a_atoms;
  p1.a_cols = a_cols;
  p1.a_cols_atoms = a_cols_atoms;
  CUtensorMap tsa, tsb;
  if ((rc = tmap_atoms(&tsa, xp_atoms, (uint64_t)R / 128 + E, H / 128))) return rc;
  if ((rc = tmap_atoms(&tsb, w1_scale, (uint64_t)E * 2 * F / 128, H / 128))) return rc;
  if ((rc = launch_gemm_mx_pair<MXEPI_SWIGLU_Q>(ta, tb, tsa, tsb, p1, st))) return rc;
  // fc2: A = a codes [R, F], B = w2 codes [E, H, F]
  if ((rc = tmap_chunks(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, 1, R, F, 1, 128, mx2::kChunks))) return rc;
  if ((rc = tmap_chunks(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w2, E, H, F, 1, 128, mx2::kChunks))) return rc;
  MxGemmParams p2{};
  p2.g = base_params(split_sizes, E);
  p2.g.M = R;
  p2.g.N = H;
  p2.g.K = F;
  p2.g.out = yp;
  p2.g.ldo = H;
  p2.g.out_f32 = out_f32;
  p2.a_atoms = a_atoms;
  p2.b_atoms = w2_scale;
  p2.b_rows = H;
  p2.out_atoms = nullptr;
  if ((rc = tmap_atoms(&tsa, a_atoms, (uint64_t)R / 128 + E, F / 128))) return rc;
  if ((rc = tmap_atoms(&tsb, w2_scale, (uint64_t)E * H / 128, F / 128))) return rc;
  p2.g.row_token = row_token;
  p2.g.out32 = out32;
  return launch_gemm_mx_pair<MXEPI_STORE>(ta, tb, tsa, tsb, p2, st);
}

// Per-tensor FP8 forward: fc1 on E4M3 codes with unit block scales, the epilogue
// rescales by 1 / (s_x s_w1[e]), stores a in bf16 and keeps max |a|; a is quantised with
// one scale; fc2 on its codes, rescaled by 1 / (s_a s_w2[e]).
int grouped_mlp_fwd_fp8(const void* xp, const float* xp_scale, const int32_t* split_sizes, int E, int R, int H, int F,
                        const void* w1, const float* w1_scale, const void* w2, const float* w2_scale,
                        const float* probs_perm, void* yp, int out_f32, void* saved, void* ws, cudaStream_t st,
                        const int32_t* row_token, float* out32) {
  if ((H % 128) || (F % 128)) return MOE_ERR_UNSUPPORTED;
  if (!xp_scale || !w1_scale || !w2_scale) return MOE_ERR_INVALID_ARG;
  uint8_t* unit = reinterpret_cast<uint8_t*>(ws);
  const size_t ub = fp8_unit_atoms_bytes(E, R, H, F);
  unsigned int* amax = reinterpret_cast<unsigned int*>(unit + ub);
  uint16_t* a_bf = reinterpret_cast<uint16_t*>(unit + ub + 256);
  uint8_t* a_codes = reinterpret_cast<uint8_t*>(a_bf) + align_up((size_t)R * F * 2, 256);
  uint16_t* h_buf = nullptr;
  if (saved) {
    h_buf = reinterpret_cast<uint16_t*>(saved);
    a_codes = reinterpret_cast<uint8_t*>(saved) + align_up((size_t)R * 2 * F * 2, 256);
  }
  float* a_scale = reinterpret_cast<float*>(a_codes + align_up((size_t)R * F, 256));
  if (cudaMemsetAsync(unit, 127, ub, st) != cudaSuccess || cudaMemsetAsync(amax, 0, 4, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  CUtensorMap ta, tb, tsa, tsb;
  int rc;
  // fc1: A = xp codes [R, H], B = w1 codes [E, 2F, H] (both K-major)
  if ((rc = tmap_chunks(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, xp, 1, R, H, 1, 128, mx2::kChunks))) return rc;
  if ((rc = tmap_chunks(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w1, E, 2 * F, H, 1, 128, mx2::kChunks))) return rc;
  if ((rc = tmap_atoms(&tsa, unit, (uint64_t)R / 128 + E, H / 128))) return rc;
  if ((rc = tmap_atoms(&tsb, unit, (uint64_t)E * 2 * F / 128, H / 128))) return rc;
  MxGemmParams p1{};
  p1.g = base_params(split_sizes, E);
  p1.g.M = R;
  p1.g.N = F;
  p1.g.K = H;
  p1.g.out = a_bf;
  p1.g.ldo = F;
  p1.g.out2 = h_buf;
  p1.g.ldo2 = 2 * F;
  p1.g.probs = probs_perm;
  p1.g.F = F;
  p1.a_atoms = unit;
  p1.b_atoms = unit;
  p1.b_rows = 2 * F;
  p1.deq_a = xp_scale;
  p1.deq_b = w1_scale;
  p1.amax_out = amax;
  if ((rc = launch_gemm_mx_pair<MXEPI_SWIGLU_F8>(ta, tb, tsa, tsb, p1, st))) return rc;
  // a: one E4M3 scale over all rows
  if ((rc = fp8_scale_launch(amax, 1, 0, a_scale, st))) return rc;
  if ((rc = fp8_cast_launch(a_bf, 1, (long long)R * F, a_scale, 0, a_codes, st))) return rc;
  // fc2: A = a codes [R, F], B = w2 codes [E, H, F]
  if ((rc = tmap_chunks(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, 1, R, F, 1, 128, mx2::kChunks))) return rc;
  if ((rc = tmap_chunks(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w2, E, H, F, 1, 128, mx2::kChunks))) return rc;
  if ((rc = tmap_atoms(&tsa, unit, (uint64_t)R / 128 + E, F / 128))) return rc;
  if ((rc = tmap_atoms(&tsb, unit, (uint64_t)E * H / 128, F / 128))) return rc;
  MxGemmParams p2{};
  p2.g = base_params(split_sizes, E);
  p2.g.M = R;
  p2.g.N = H;
  p2.g.K = F;
  p2.g.out = yp;
  p2.g.ldo = H;
  p2.g.out_f32 = out_f32;
  p2.g.row_token = row_token;
  p2.g.out32 = out32;
  p2.a_atoms = unit;
  p2.b_atoms = unit;
  p2.b_rows = H;
  p2.deq_a = a_scale;
  p2.deq_b = w2_scale;
  return launch_gemm_mx_pair<MXEPI_STORE>(ta, tb, tsa, tsb, p2, st);
}

// The forward; with row_token, fc2's rows are added into out32[row_token[r]] (fused
// combine) instead of being stored to yp.
int grouped_mlp_fwd_impl(const void* xp, const uint8_t* xp_scale, const int32_t* split_sizes, int E, int R, int H,
                         int F, const void* w1, const uint8_t* w1_scale, const void* w2, const uint8_t* w2_scale,
                         const float* probs_perm, int precision, void* yp, void* saved, void* ws, size_t ws_bytes,
                         cudaStream_t st, const int32_t* row_token, float* out32) {
  const int out_f32 = (precision & MOE_OUT_F32) ? 1 : 0;
  precision &= ~MOE_OUT_F32;
  if (E < 1 || E > gg::kMaxE || R < 0 || H < 64 || F < 128) return MOE_ERR_INVALID_ARG;
  if (precision != MOE_BF16 && precision != MOE_MXFP8 && precision != MOE_FP8) return MOE_ERR_INVALID_ARG;
  if ((H % 64) || (F % 128)) return MOE_ERR_UNSUPPORTED;
  if (R == 0) return MOE_OK;
  if (!xp || !split_sizes || !w1 || !w2 || (!yp && !row_token) || !ws) return MOE_ERR_INVALID_ARG;
  const int training = saved != nullptr;
  if (ws_bytes < grouped_mlp_workspace_size(E, R, H, F, precision, training)) return MOE_ERR_INVALID_ARG;
  if (precision == MOE_FP8)
    return grouped_mlp_fwd_fp8(xp, reinterpret_cast<const float*>(xp_scale), split_sizes, E, R, H, F, w1,
                               reinterpret_cast<const float*>(w1_scale), w2, reinterpret_cast<const float*>(w2_scale),
                               probs_perm, yp, out_f32, saved, ws, st, row_token, out32);
  if (precision == MOE_MXFP8)
    return grouped_mlp_fwd_mxfp8(xp, xp_scale, split_sizes, E, R, H, F, w1, w1_scale, w2, w2_scale, probs_perm, yp,
                                 out_f32, saved, ws, st, row_token, out32);

  uint16_t* h_buf = nullptr;
  uint16_t* a_buf = reinterpret_cast<uint16_t*>(ws);
  if (training) {
    h_buf = reinterpret_cast<uint16_t*>(saved);
    a_buf = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(saved) + align_up((size_t)R * 2 * F * 2, 256));
  }
  CUtensorMap ta, tb;
  int rc;
  // fc1: A = xp [R, H] (K-major), B = w1 [E, H, 2F] (N contiguous: MN-major)
  if ((rc = tmap_chunks(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, xp, 1, R, H, 2))) return rc;
  if ((rc = tmap_chunks(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w1, E, H, 2 * F, 2))) return rc;
  GemmParams p1 = base_params(split_sizes, E);
  p1.M = R;
  p1.N = F;
  p1.K = H;
  p1.out = a_buf;
  p1.ldo = F;
  p1.out2 = h_buf;
  p1.ldo2 = 2 * F;
  p1.probs = probs_perm;
  p1.F = F;
  if ((rc = launch_gemm_pair<true, EPI_SWIGLU>(ta, tb, p1, st))) return rc;
  // fc2: A = a [R, F] (K-major), B = w2 [E, F, H] (MN-major)
  if ((rc = tmap_chunks(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a_buf, 1, R, F, 2))) return rc;
  if ((rc = tmap_chunks(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w2, E, F, H, 2))) return rc;
  GemmParams p2 = base_params(split_sizes, E);
  p2.M = R;
  p2.N = H;
  p2.K = F;
  p2.out = yp;
  p2.ldo = H;
  p2.out_f32 = out_f32;
  p2.row_token = row_token;
  p2.out32 = out32;
  return launch_gemm_pair<true, EPI_STORE>(ta, tb, p2, st);
}

}  // namespace

extern "C" {

int grouped_mlp_fwd(const void* xp, const uint8_t* xp_scale, const int32_t* split_sizes, int E, int R, int H, int F,
                    const void* w1, const uint8_t* w1_scale, const void* w2, const uint8_t* w2_scale,
                    const float* probs_perm, int precision, void* yp, void* saved, void* ws, size_t ws_bytes,
                    void* stream) {
  return grouped_mlp_fwd_impl(xp, xp_scale, split_sizes, E, R, H, F, w1, w1_scale, w2, w2_scale, probs_perm,
                              precision, yp, saved, ws, ws_bytes, as_stream(stream), nullptr, nullptr);
}

size_t grouped_mlp_fwd_combine_workspace_size(int E, int R, int H, int F, int precision, int training, int T) {
  if (R < 0 || F < 0 || T < 0) return 0;
  return grouped_mlp_workspace_size(E, R, H, F, precision, training) + align_up((size_t)T * H * 4, 256) +
         align_up((size_t)R * 4, 256);
}

int grouped_mlp_fwd_combine(const void* xp, const uint8_t* xp_scale, const int32_t* split_sizes, int E, int R, int H,
                            int F, const void* w1, const uint8_t* w1_scale, const void* w2, const uint8_t* w2_scale,
                            const float* probs_perm, int precision, const int32_t* row_map, int T, int k,
                            uint16_t* out, void* saved, void* ws, size_t ws_bytes, void* stream) {
  if (T < 0 || k < 1 || k > 32 || (long long)T * k != R || (precision & MOE_OUT_F32)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!row_map || !out || !ws) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(out) & 15) || (H % 8)) return MOE_ERR_INVALID_ARG;
  const int training = saved != nullptr;
  if (ws_bytes < grouped_mlp_fwd_combine_workspace_size(E, R, H, F, precision, training, T))
    return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  const size_t base = grouped_mlp_workspace_size(E, R, H, F, precision, training);
  float* out32 = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + base);
  int32_t* row_token =
      reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(out32) + align_up((size_t)T * H * 4, 256));
  if (cudaMemsetAsync(out32, 0, (size_t)T * H * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
  row_token_kernel<<<std::min((R + 255) / 256, device_props().sm_count * 8), 256, 0, st>>>(row_map, R, k, row_token);
  count_launch();
  int rc = launch_status();
  if (rc) return rc;
  rc = grouped_mlp_fwd_impl(xp, xp_scale, split_sizes, E, R, H, F, w1, w1_scale, w2, w2_scale, probs_perm, precision,
                            nullptr, saved, ws, base, st, row_token, out32);
  if (rc) return rc;
  const long long n8 = (long long)T * H / 8;
  f32_to_bf16_kernel<<<(int)std::min<long long>((n8 + 255) / 256, (long long)device_props().sm_count * 8), 256, 0,
                       st>>>(reinterpret_cast<const float4*>(out32), n8, reinterpret_cast<uint4*>(out));
  count_launch();
  return launch_status();
}

}  // extern "C"

namespace {

// Backward workspace parts (each 256-byte aligned, in this order):
//   0 dh bf16 [R, 2F] (BF16 only);  2 dprob partial sums [ceil(F/256)][R] fp32;
//   MXFP8 only, quantised operands:
//   3 w2 codes [E, F, H] + scale atoms;  4 w1 codes [E, H, 2F] + atoms;
//   5 dy codes [R, H] + plain scales + atoms (along H);  6 dy codes + atoms (along rows);
//   7 a codes [R, F] + atoms (rows);  8 dh codes [R, 2F] + atoms (along 2F);
//   9 dh codes + atoms (rows);  10 xp codes [R, H] + atoms (rows).
// (Part 1 is no longer used: the MXFP8 fc2-dgrad epilogue quantises a and dh itself.)
size_t bwd_part_bytes(int part, int E, int R, int H, int F, int precision) {
  const size_t r = (size_t)R, e = (size_t)E, h = (size_t)H, f = (size_t)F;
  if (precision == MOE_FP8) {
    // 0 dh bf16; 2 dprob partials; 3 w2 codes [E, F, H] + E scales; 4 w1 codes
    // [E, H, 2F] + E scales; 5 dy codes [R, H] + scale; 8 dh codes [R, 2F] + scale;
    // 10 xp codes [R, H] + scale; 11 max words + unit block scales
    switch (part) {
      case 0: return align_up(r * 2 * f * 2, 256);
      case 2: return align_up((size_t)(2 * ((F + gg::BN - 1) / gg::BN)) * r * 4, 256);
      case 3: return align_up(e * f * h, 256) + align_up(e * 4, 256);
      case 4: return align_up(e * h * 2 * f, 256) + align_up(e * 4, 256);
      case 5: return align_up(r * h, 256) + 256;
      case 8: return align_up(r * 2 * f, 256) + 256;
      case 10: return align_up(r * h, 256) + 256;
      case 11: return align_up(e * 4 + 16, 256) + fp8_unit_atoms_bytes(E, R, H, F);
      default: return 0;
    }
  }
  const bool mx = precision == MOE_MXFP8;
  switch (part) {
    case 0: return mx ? 0 : align_up(r * 2 * f * 2, 256);
    case 2: return align_up((size_t)(2 * ((F + gg::BN - 1) / gg::BN)) * r * 4, 256);
    case 3: return mx ? align_up(e * f * h, 256) + align_up(e * f * h / 32, 256) : 0;
    case 4: return mx ? align_up(e * h * 2 * f, 256) + align_up(e * h * 2 * f / 32, 256) : 0;
    case 5: return mx ? align_up(r * h, 256) + align_up(r * h / 32, 256) + mma_atoms_bytes(E, R, H) : 0;
    case 6: return mx ? align_up(r * h, 256) + mma_atoms_bytes(E, R, H) : 0;
    case 7: return 0;   // (a along rows now comes from the forward's saved buffer)
    case 8: return mx ? align_up(r * 2 * f, 256) + mma_atoms_bytes(E, R, 2 * F) : 0;
    case 9: return mx ? align_up(r * 2 * f, 256) + mma_atoms_bytes(E, R, 2 * F) : 0;
    case 10: return mx ? align_up(r * h, 256) + mma_atoms_bytes(E, R, H) : 0;
    default: return 0;
  }
}

size_t bwd_part_offset(int part, int E, int R, int H, int F, int precision) {
  size_t off = 0;
  for (int i = 0; i < part; ++i) off += bwd_part_bytes(i, E, R, H, F, precision);
  return off;
}

}  // namespace

extern "C" {

size_t grouped_mlp_bwd_workspace_size(int E, int R, int H, int F, int precision) {
  if (R < 0 || F < 0 || E < 1) return 0;
  return bwd_part_offset(12, E, R, H, F, precision) + 256;
}

size_t grouped_mlp_bwd_workspace_offset(int E, int R, int H, int F, int precision, int part) {
  if (R < 0 || F < 0 || E < 1) return (size_t)-1;
  const bool ok = precision == MOE_MXFP8 ? (part == 8 || part == 9)
                  : precision == MOE_FP8 ? (part == 0 || part == 8)
                                         : part == 0;
  return ok ? bwd_part_offset(part, E, R, H, F, precision) : (size_t)-1;
}

}  // extern "C"

namespace {

// Per-tensor FP8 backward: dy and dh in E5M2 (one scale each), xp, the saved a and the
// weights (one scale per expert) in E4M3; per-tensor codes serve both orientations, so
// the weight-gradient GEMMs read the same code arrays MN-major.
int grouped_mlp_bwd_fp8(const void* dy_perm, const int32_t* split_sizes, int E, int R, int H, int F, const void* xp,
                        const void* w1, const void* w2, const float* probs_perm, const void* saved, uint16_t* dxp,
                        uint16_t* dw1, uint16_t* dw2, float* dprobs_perm, void* ws, cudaStream_t st) {
  if ((H % 128) || (F % 128)) return MOE_ERR_UNSUPPORTED;
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  auto part = [&](int i) { return base + bwd_part_offset(i, E, R, H, F, MOE_FP8); };
  uint16_t* dh = reinterpret_cast<uint16_t*>(part(0));
  float* dpart = reinterpret_cast<float*>(part(2));
  const size_t efh = (size_t)E * F * H;
  uint8_t* w2q = part(3);
  float* s_w2 = reinterpret_cast<float*>(w2q + align_up(efh, 256));
  uint8_t* w1q = part(4);
  float* s_w1 = reinterpret_cast<float*>(w1q + align_up(efh * 2, 256));
  uint8_t* dyq = part(5);
  float* s_dy = reinterpret_cast<float*>(dyq + align_up((size_t)R * H, 256));
  uint8_t* dhq = part(8);
  float* s_dh = reinterpret_cast<float*>(dhq + align_up((size_t)R * 2 * F, 256));
  uint8_t* xq = part(10);
  float* s_x = reinterpret_cast<float*>(xq + align_up((size_t)R * H, 256));
  unsigned int* amax = reinterpret_cast<unsigned int*>(part(11));           // [E] (+ one for dh)
  uint8_t* unit = part(11) + align_up((size_t)E * 4 + 16, 256);
  const uint8_t* a_codes = reinterpret_cast<const uint8_t*>(saved) + align_up((size_t)R * 2 * F * 2, 256);
  const float* a_scale = reinterpret_cast<const float*>(a_codes + align_up((size_t)R * F, 256));
  const uint16_t* h_saved = reinterpret_cast<const uint16_t*>(saved);
  const int nparts = 2 * ((F + gg::BN - 1) / gg::BN);
  const uint32_t A_E5M2 = 1u << 7, B_E5M2 = 1u << 10;
  int rc;
  if (cudaMemsetAsync(unit, 127, fp8_unit_atoms_bytes(E, R, H, F), st) != cudaSuccess) return MOE_ERR_CUDA;
  // operands: weights per expert (their own layout: K-major for the data gradients),
  // dy and xp over all rows
  if ((rc = fp8_quantize_launch(w2, E, (long long)F * H, 0, w2q, s_w2, amax, st))) return rc;
  if ((rc = fp8_quantize_launch(w1, E, (long long)H * 2 * F, 0, w1q, s_w1, amax, st))) return rc;
  if ((rc = fp8_quantize_launch(dy_perm, 1, (long long)R * H, 1, dyq, s_dy, amax, st))) return rc;
  if ((rc = fp8_quantize_launch(xp, 1, (long long)R * H, 0, xq, s_x, amax, st))) return rc;
  CUtensorMap ta, tb, tsa, tsb;
  // fc2 dgrad + SwiGLU backward: A = dy (E5M2) [R, H], B = w2 (E4M3) [E, F, H]; dh bf16
  if ((rc = tmap_chunks(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, dyq, 1, R, H, 1, 128, mx2::kChunks))) return rc;
  if ((rc = tmap_chunks(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w2q, E, F, H, 1, 128, mx2::kChunks))) return rc;
  if ((rc = tmap_atoms(&tsa, unit, (uint64_t)R / 128 + E, H / 128))) return rc;
  if ((rc = tmap_atoms(&tsb, unit, (uint64_t)E * F / 128, H / 128))) return rc;
  if (cudaMemsetAsync(amax, 0, 4, st) != cudaSuccess) return MOE_ERR_CUDA;
  MxGemmParams p{};
  p.g = base_params(split_sizes, E);
  p.g.M = R;
  p.g.N = F;
  p.g.K = H;
  p.g.out2 = dh;
  p.g.ldo2 = 2 * F;
  p.g.aux = h_saved;
  p.g.ld_aux = 2 * F;
  p.g.probs = probs_perm;
  p.g.dprob_part = dpart;
  p.g.F = F;
  p.a_atoms = unit;
  p.b_atoms = unit;
  p.b_rows = F;
  p.ab_fmt = A_E5M2;
  p.deq_a = s_dy;
  p.deq_b = s_w2;
  p.amax_out = amax;
  if ((rc = launch_gemm_mx_pair<MXEPI_DSWIGLU_F8>(ta, tb, tsa, tsb, p, st))) return rc;
  if (dprobs_perm) {
    const int grid = std::min((R + 255) / 256, device_props().sm_count * 4);
    reduce_dprob_kernel<<<grid, 256, 0, st>>>(dpart, nparts, R, dprobs_perm);
    count_launch();
    if ((rc = launch_status())) return rc;
  }
  // dh: one E5M2 scale
  if ((rc = fp8_scale_launch(amax, 1, 1, s_dh, st))) return rc;
  if ((rc = fp8_cast_launch(dh, 1, (long long)R * 2 * F, s_dh, 1, dhq, st))) return rc;
  // fc2 wgrad: dw2[e] = a_e^T dy_e, A = a codes (E4M3) [R, F], B = dy codes (E5M2) [R, H]
  const uint64_t n_unit = fp8_unit_atoms_bytes(E, R, H, F) / 512;
  p = MxGemmParams{};
  p.g = base_params(split_sizes, E);
  p.g.M = F;
  p.g.N = H;
  p.g.out = dw2;
  p.g.ldo = H;
  p.g.out_batch = (long long)F * H;
  p.a_atoms = unit;
  p.b_atoms = unit;
  p.b_rows = H;
  p.ab_fmt = B_E5M2;
  p.deq_a = a_scale;
  p.deq_b = s_dy;
  if ((rc = launch_wgrad_mx_pair(a_codes, unit, n_unit, dyq, unit, n_unit, R, p, st))) return rc;
  // fc1 dgrad: dxp = dh w1[e]^T, A = dh codes (E5M2) [R, 2F], B = w1 codes [E, H, 2F]
  if ((rc = tmap_chunks(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, dhq, 1, R, 2 * F, 1, 128, mx2::kChunks))) return rc;
  if ((rc = tmap_chunks(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w1q, E, H, 2 * F, 1, 128, mx2::kChunks))) return rc;
  if ((rc = tmap_atoms(&tsa, unit, (uint64_t)R / 128 + E, 2 * F / 128))) return rc;
  if ((rc = tmap_atoms(&tsb, unit, (uint64_t)E * H / 128, 2 * F / 128))) return rc;
  p = MxGemmParams{};
  p.g = base_params(split_sizes, E);
  p.g.M = R;
  p.g.N = H;
  p.g.K = 2 * F;
  p.g.out = dxp;
  p.g.ldo = H;
  p.a_atoms = unit;
  p.b_atoms = unit;
  p.b_rows = H;
  p.ab_fmt = A_E5M2;
  p.deq_a = s_dh;
  p.deq_b = s_w1;
  if ((rc = launch_gemm_mx_pair<MXEPI_STORE>(ta, tb, tsa, tsb, p, st))) return rc;
  // fc1 wgrad: dw1[e] = xp_e^T dh_e, A = xp codes (E4M3) [R, H], B = dh codes (E5M2)
  p = MxGemmParams{};
  p.g = base_params(split_sizes, E);
  p.g.M = H;
  p.g.N = 2 * F;
  p.g.out = dw1;
  p.g.ldo = 2 * F;
  p.g.out_batch = (long long)H * 2 * F;
  p.a_atoms = unit;
  p.b_atoms = unit;
  p.b_rows = 2 * F;
  p.ab_fmt = B_E5M2;
  p.deq_a = s_x;
  p.deq_b = s_dh;
  return launch_wgrad_mx_pair(xq, unit, n_unit, dhq, unit, n_unit, R, p, st);
}

// q: operands the caller quantised already (NULL pairs, or q == NULL: quantised here into
// the workspace from dy_perm, xp, w1, w2).
int grouped_mlp_bwd_mxfp8(const moe_mxfp8_bwd_operands* q, const void* dy_perm, const int32_t* split_sizes, int E,
                          int R, int H, int F, const void* xp, const void* w1, const void* w2, const float* probs_perm,
                          const void* saved, uint16_t* dxp, uint16_t* dw1, uint16_t* dw2, float* dprobs_perm,
                          void* ws, cudaStream_t st) {
  if ((H % 128) || (F % 128)) return MOE_ERR_UNSUPPORTED;
  const moe_mxfp8_bwd_operands none{};
  if (!q) q = &none;
  const bool have_w2 = q->w2_rows && q->w2_rows_atoms, have_w1 = q->w1_rows && q->w1_rows_atoms;
  const bool have_dyr = q->dy_rows && q->dy_rows_atoms, have_dyc = q->dy_cols && q->dy_cols_atoms;
  const bool have_xc = q->xp_cols && q->xp_cols_atoms;
  if ((!have_w2 && !w2) || (!have_w1 && !w1) || ((!have_dyr || !have_dyc) && !dy_perm) || (!have_xc && !xp))
    return MOE_ERR_INVALID_ARG;
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  auto part = [&](int i) { return base + bwd_part_offset(i, E, R, H, F, MOE_MXFP8); };
  float* dpart = reinterpret_cast<float*>(part(2));
  const size_t efh = (size_t)E * F * H;
  uint8_t* w2q_ws = part(3);
  uint8_t* w2a_ws = w2q_ws + align_up(efh, 256);
  uint8_t* w1q_ws = part(4);
  uint8_t* w1a_ws = w1q_ws + align_up(efh * 2, 256);
  uint8_t* dyr_ws = part(5);
  uint8_t* dyr_s = dyr_ws + align_up((size_t)R * H, 256);
  uint8_t* dyr_a_ws = dyr_s + align_up((size_t)R * H / 32, 256);
  uint8_t* dyc_ws = part(6);
  uint8_t* dyc_a_ws = dyc_ws + align_up((size_t)R * H, 256);
  const uint8_t* w2q = have_w2 ? q->w2_rows : w2q_ws;
  const uint8_t* w2a = have_w2 ? q->w2_rows_atoms : w2a_ws;
  const uint8_t* w1q = have_w1 ? q->w1_rows : w1q_ws;
  const uint8_t* w1a = have_w1 ? q->w1_rows_atoms : w1a_ws;
  const uint8_t* dyr = have_dyr ? q->dy_rows : dyr_ws;
  const uint8_t* dyr_a = have_dyr ? q->dy_rows_atoms : dyr_a_ws;
  const uint8_t* dyc = have_dyc ? q->dy_cols : dyc_ws;
  const uint8_t* dyc_a = have_dyc ? q->dy_cols_atoms : dyc_a_ws;
  // a along the expert's rows: quantised by the forward's fc1 epilogue into `saved`
  const uint8_t* ac = reinterpret_cast<const uint8_t*>(saved) + align_up((size_t)R * 2 * F * 2, 256) +
                      align_up((size_t)R * F, 256) + mma_atoms_bytes(E, R, F);
  const uint8_t* ac_a = ac + align_up((size_t)R * F, 256);
  uint8_t* dhr = part(8);
  uint8_t* dhr_a = dhr + align_up((size_t)R * 2 * F, 256);
  uint8_t* dhc = part(9);
  uint8_t* dhc_a = dhc + align_up((size_t)R * 2 * F, 256);
  uint8_t* xc_ws = part(10);
  uint8_t* xc_a_ws = xc_ws + align_up((size_t)R * H, 256);
  const uint8_t* xc = have_xc ? q->xp_cols : xc_ws;
  const uint8_t* xc_a = have_xc ? q->xp_cols_atoms : xc_a_ws;
  const uint16_t* h_saved = reinterpret_cast<const uint16_t*>(saved);
  const int nparts = 2 * ((F + gg::BN - 1) / gg::BN);   // one partial per N-tile half
  int rc;
  // weights along their other axis (the masters change every optimizer step)
  if (!have_w2 && (rc = quant_rows_launch(w2, (long long)E * F, H, 1, w2q_ws, w2a_ws, st))) return rc;
  if (!have_w1 && (rc = quant_rows_launch(w1, (long long)E * H, 2 * F, 1, w1q_ws, w1a_ws, st))) return rc;
  // dy along H (fc2 dgrad) and along rows (fc2 wgrad)
  if (!have_dyr) {
    if ((rc = quant_rows_launch(dy_perm, R, H, 0, dyr_ws, dyr_s, st))) return rc;
    if ((rc = scales_to_atoms_launch(dyr_s, split_sizes, E, R, H, dyr_a_ws, st))) return rc;
  }
  if (!have_dyc && (rc = quant_cols_grouped_launch(dy_perm, R, H, split_sizes, E, dyc_ws, dyc_a_ws, st))) return rc;
  CUtensorMap ta, tb;
  // fc2 dgrad + SwiGLU backward: A = dy codes [R, H], B = w2 codes [E, F, H] (N = F)
  if ((rc = tmap_chunks(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, dyr, 1, R, H, 1, 128, mx2::kChunks))) return rc;
  if ((rc = tmap_chunks(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w2q, E, F, H, 1, 128, mx2::kChunks))) return rc;
  MxGemmParams p{};
  p.g = base_params(split_sizes, E);
  p.g.M = R;
  p.g.N = F;
  p.g.K = H;
  p.g.aux = h_saved;
  p.g.ld_aux = 2 * F;
  p.g.probs = probs_perm;
  p.g.dprob_part = dpart;
  p.g.F = F;
  p.a_atoms = dyr_a;
  p.b_atoms = w2a;
  p.b_rows = F;
  p.out_atoms = nullptr;
  // the epilogue quantises dh for the two GEMMs of fc1 that follow
  p.dh_rows = dhr;
  p.dh_rows_atoms = dhr_a;
  p.dh_cols = dhc;
  p.dh_cols_atoms = dhc_a;
  CUtensorMap tsa, tsb;
  if ((rc = tmap_atoms(&tsa, dyr_a, (uint64_t)R / 128 + E, H / 128))) return rc;
  if ((rc = tmap_atoms(&tsb, w2a, (uint64_t)E * F / 128, H / 128))) return rc;
  // the saved h, staged into shared memory for the epilogue by TMA (32-column strips)
  CUtensorMap th;
  if ((rc = make_tmap(&th, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h_saved, 2 * F, R, 1, (uint64_t)4 * F,
                      (uint64_t)R * 4 * F, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B)))
    return rc;
  if ((rc = launch_gemm_mx_pair<MXEPI_DSWIGLU>(ta, tb, tsa, tsb, p, st, &th))) return rc;
  if (dprobs_perm) {
    const int grid = std::min((R + 255) / 256, device_props().sm_count * 4);
    reduce_dprob_kernel<<<grid, 256, 0, st>>>(dpart, nparts, R, dprobs_perm);
    count_launch();
    if ((rc = launch_status())) return rc;
  }
  // xp along its rows for the fc1 weight gradient
  if (!have_xc && (rc = quant_cols_grouped_launch(xp, R, H, split_sizes, E, xc_ws, xc_a_ws, st))) return rc;
  // fc2 wgrad: dw2[e] = a_e^T dy_e (MN-major codes, contraction over the expert's rows)
  const uint64_t kgs = (uint64_t)R / 128 + E;   // bound on the experts' 128-row k-groups
  p.g = base_params(split_sizes, E);
  p.g.M = F;
  p.g.N = H;
  p.g.out = dw2;
  p.g.ldo = H;
  p.g.out_batch = (long long)F * H;
  p.a_atoms = ac_a;
  p.b_atoms = dyc_a;
  p.b_rows = H;
  if ((rc = launch_wgrad_mx_pair(ac, ac_a, kgs * (F / 128), dyc, dyc_a, kgs * (H / 128), R, p, st))) return rc;
  // fc1 dgrad: dxp = dh w1[e]^T. A = dh codes [R, 2F], B = w1 codes [E, H, 2F] (N = H)
  if ((rc = tmap_chunks(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, dhr, 1, R, 2 * F, 1, 128, mx2::kChunks))) return rc;
  if ((rc = tmap_chunks(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w1q, E, H, 2 * F, 1, 128, mx2::kChunks))) return rc;
  p.g = base_params(split_sizes, E);
  p.g.M = R;
  p.g.N = H;
  p.g.K = 2 * F;
  p.g.out = dxp;
  p.g.ldo = H;
  p.a_atoms = dhr_a;
  p.b_atoms = w1a;
  p.b_rows = H;
  if ((rc = tmap_atoms(&tsa, dhr_a, (uint64_t)R / 128 + E, 2 * F / 128))) return rc;
  if ((rc = tmap_atoms(&tsb, w1a, (uint64_t)E * H / 128, 2 * F / 128))) return rc;
  if ((rc = launch_gemm_mx_pair<MXEPI_STORE>(ta, tb, tsa, tsb, p, st))) return rc;
  // fc1 wgrad: dw1[e] = xp_e^T dh_e
  p.g = base_params(split_sizes, E);
  p.g.M = H;
  p.g.N = 2 * F;
  p.g.out = dw1;
  p.g.ldo = 2 * F;
  p.g.out_batch = (long long)H * 2 * F;
  p.a_atoms = xc_a;
  p.b_atoms = dhc_a;
  p.b_rows = 2 * F;
  return launch_wgrad_mx_pair(xc, xc_a, kgs * (H / 128), dhc, dhc_a, kgs * (2 * F / 128), R, p, st);
}

}  // namespace

extern "C" {

int grouped_mlp_bwd(const void* dy_perm, const int32_t* split_sizes, int E, int R, int H, int F, const void* xp,
                    const void* w1, const void* w2, const float* probs_perm, int precision, const void* saved,
                    uint16_t* dxp, uint16_t* dw1, uint16_t* dw2, float* dprobs_perm, void* ws, size_t ws_bytes,
                    void* stream) {
  if (E < 1 || E > gg::kMaxE || R < 0 || H < 64 || F < 128) return MOE_ERR_INVALID_ARG;
  if ((H % 64) || (F % 128)) return MOE_ERR_UNSUPPORTED;
  if (precision != MOE_BF16 && precision != MOE_MXFP8 && precision != MOE_FP8) return MOE_ERR_INVALID_ARG;
  if (!split_sizes || !w1 || !w2 || !dw1 || !dw2) return MOE_ERR_INVALID_ARG;
  if (R > 0 && (!dy_perm || !xp || !saved || !dxp || !ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < grouped_mlp_bwd_workspace_size(E, R, H, F, precision)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  if (R == 0) {
    if (cudaMemsetAsync(dw1, 0, (size_t)E * H * 2 * F * 2, st) != cudaSuccess ||
        cudaMemsetAsync(dw2, 0, (size_t)E * F * H * 2, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (precision == MOE_MXFP8)
    return grouped_mlp_bwd_mxfp8(nullptr, dy_perm, split_sizes, E, R, H, F, xp, w1, w2, probs_perm, saved, dxp, dw1, dw2,
                                 dprobs_perm, ws, st);
  if (precision == MOE_FP8)
    return grouped_mlp_bwd_fp8(dy_perm, split_sizes, E, R, H, F, xp, w1, w2, probs_perm, saved, dxp, dw1, dw2,
                               dprobs_perm, ws, st);
  const uint16_t* h_buf = reinterpret_cast<const uint16_t*>(saved);
  const uint16_t* a_buf =
      reinterpret_cast<const uint16_t*>(reinterpret_cast<const uint8_t*>(saved) + align_up((size_t)R * 2 * F * 2, 256));
  uint16_t* dh = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(ws) + bwd_part_offset(0, E, R, H, F, MOE_BF16));
  float* dpart = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + bwd_part_offset(2, E, R, H, F, MOE_BF16));
  const int nparts = 2 * ((F + gg::BN - 1) / gg::BN);   // one partial per N-tile half

  CUtensorMap ta, tb;
  int rc;
  // fc2 dgrad + SwiGLU backward: A = dy [R, H] (K-major), B = w2 [E, F, H] read as [E, N=F, K=H] (K-major)
  if ((rc = tmap_chunks(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dy_perm, 1, R, H, 2))) return rc;
  if ((rc = tmap_chunks(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w2, E, F, H, 2))) return rc;
  GemmParams p = base_params(split_sizes, E);
  p.M = R;
  p.N = F;
  p.K = H;
  p.out2 = dh;
  p.ldo2 = 2 * F;
  p.probs = probs_perm;
  p.aux = h_buf;
  p.ld_aux = 2 * F;
  p.dprob_part = dpart;
  p.F = F;
  // the saved h, staged into shared memory for the epilogue by TMA (32-column strips)
  CUtensorMap th;
  if ((rc = make_tmap(&th, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, h_buf, 2 * F, R, 1, (uint64_t)4 * F,
                      (uint64_t)R * 4 * F, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B)))
    return rc;
  if ((rc = launch_gemm_pair<false, EPI_DSWIGLU>(ta, tb, p, st, &th))) return rc;
  if (dprobs_perm) {
    const int grid = std::min((R + 255) / 256, device_props().sm_count * 4);
    reduce_dprob_kernel<<<grid, 256, 0, st>>>(dpart, nparts, R, dprobs_perm);
    count_launch();
    if ((rc = launch_status())) return rc;
  }
  // fc2 wgrad: dw2[e] = a_e^T dy_e. A = a [R, F] (rows = K, MN-major), B = dy [R, H] (MN-major)
  if ((rc = tmap_chunks(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a_buf, 1, R, F, 2, kp::BK, 2))) return rc;
  if ((rc = tmap_chunks(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dy_perm, 1, R, H, 2, kp::BK, 2))) return rc;
  p = base_params(split_sizes, E);
  p.M = F;
  p.N = H;
  p.out = dw2;
  p.ldo = H;
  p.out_batch = (long long)F * H;
  if ((rc = launch_wgrad_pair(ta, tb, p, st))) return rc;
  // fc1 dgrad: dxp = dh w1[e]^T. A = dh [R, 2F] (K-major), B = w1 [E, H, 2F] read as [E, N=H, K=2F] (K-major)
  if ((rc = tmap_chunks(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dh, 1, R, 2 * F, 2))) return rc;
  if ((rc = tmap_chunks(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w1, E, H, 2 * F, 2))) return rc;
  p = base_params(split_sizes, E);
  p.M = R;
  p.N = H;
  p.K = 2 * F;
  p.out = dxp;
  p.ldo = H;
  if ((rc = launch_gemm_pair<false, EPI_STORE>(ta, tb, p, st))) return rc;
  // fc1 wgrad: dw1[e] = xp_e^T dh_e. A = xp [R, H] (MN-major), B = dh [R, 2F] (MN-major)
  if ((rc = tmap_chunks(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, xp, 1, R, H, 2, kp::BK, 2))) return rc;
  if ((rc = tmap_chunks(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dh, 1, R, 2 * F, 2, kp::BK, 2))) return rc;
  p = base_params(split_sizes, E);
  p.M = H;
  p.N = 2 * F;
  p.out = dw1;
  p.ldo = 2 * F;
  p.out_batch = (long long)H * 2 * F;
  return launch_wgrad_pair(ta, tb, p, st);
}

int grouped_mlp_bwd_mxfp8_operands(const moe_mxfp8_bwd_operands* q, const void* dy_perm, const int32_t* split_sizes,
                                   int E, int R, int H, int F, const void* xp, const void* w1, const void* w2,
                                   const float* probs_perm, const void* saved, uint16_t* dxp, uint16_t* dw1,
                                   uint16_t* dw2, float* dprobs_perm, void* ws, size_t ws_bytes, void* stream) {
  if (E < 1 || E > gg::kMaxE || R < 0 || H < 128 || F < 128) return MOE_ERR_INVALID_ARG;
  if ((H % 128) || (F % 128)) return MOE_ERR_UNSUPPORTED;
  if (!split_sizes || !dw1 || !dw2) return MOE_ERR_INVALID_ARG;
  if (R > 0 && (!saved || !dxp || !ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < grouped_mlp_bwd_workspace_size(E, R, H, F, MOE_MXFP8)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  if (R == 0) {
    if (cudaMemsetAsync(dw1, 0, (size_t)E * H * 2 * F * 2, st) != cudaSuccess ||
        cudaMemsetAsync(dw2, 0, (size_t)E * F * H * 2, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  return grouped_mlp_bwd_mxfp8(q, dy_perm, split_sizes, E, R, H, F, xp, w1, w2, probs_perm, saved, dxp, dw1, dw2,
                               dprobs_perm, ws, st);
}

}  // extern "C"

// ---------------------------------------------------------------------------------
// Allocation-free permutation: moe_permute with its histogram table in static device
// memory instead of a caller workspace (see moe_permute_noalloc in the header).
namespace {

static __device__ __align__(256) int32_t g_permute_scratch[MOE_PERMUTE_NOALLOC_MAX_COUNTS];

// Device address of g_permute_scratch on the current device, looked up once per device
// with that device current (host code cannot use the symbol itself as a pointer).
int32_t* permute_scratch_on_current_device() {
  static int32_t* ptr[64];
  static cudaError_t err[64];
  static std::once_flag once[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::call_once(once[dev], [dev]() {
    void* p = nullptr;
    err[dev] = cudaGetSymbolAddress(&p, g_permute_scratch);
    ptr[dev] = static_cast<int32_t*>(p);
  });
  return err[dev] == cudaSuccess ? ptr[dev] : nullptr;
}

}  // namespace

extern "C" int moe_permute_noalloc(const uint16_t* x, const int32_t* idx, const float* prob, int T, int H, int E,
                                   int k, int precision, void* xp, uint8_t* xp_scale, int32_t* row_map,
                                   float* probs_perm, int32_t* split_sizes, int32_t* offsets, void* stream) {
  if (T < 0 || E < 1 || k < 1) return MOE_ERR_INVALID_ARG;
  const size_t need = permute_counts_bytes((size_t)T * k, E);
  if (need > sizeof(int32_t) * (size_t)MOE_PERMUTE_NOALLOC_MAX_COUNTS) {
    fprintf(stderr,
            "moe_permute_noalloc: T*k=%lld with E=%d needs %zu bytes of scratch; the static table holds %zu "
            "(ceil(T*k/1024)*E must be <= %d)\n",
            (long long)T * k, E, need, sizeof(int32_t) * (size_t)MOE_PERMUTE_NOALLOC_MAX_COUNTS,
            MOE_PERMUTE_NOALLOC_MAX_COUNTS);
    return MOE_ERR_UNSUPPORTED;
  }
  int32_t* scratch = permute_scratch_on_current_device();
  if (!scratch) return MOE_ERR_CUDA;
  return moe_permute(x, idx, prob, T, H, E, k, precision, xp, xp_scale, row_map, probs_perm, split_sizes, offsets,
                     scratch, sizeof(int32_t) * (size_t)MOE_PERMUTE_NOALLOC_MAX_COUNTS, stream);
}

extern "C" int mxfp8_quantize_grouped(const uint16_t* in, int R, int C, const int32_t* split_sizes, int E,
                                      uint8_t* codes, uint8_t* atoms, void* stream) {
  if (R < 0 || C < 0 || E < 1 || E > kMaxExperts) return MOE_ERR_INVALID_ARG;
  if (C % 128) return MOE_ERR_UNSUPPORTED;
  if (R == 0 || C == 0) return MOE_OK;
  if (!in || !split_sizes || !codes || !atoms) return MOE_ERR_INVALID_ARG;
  return quant_cols_grouped_launch(in, R, C, split_sizes, E, codes, atoms, as_stream(stream));
}

extern "C" size_t mxfp8_grouped_atoms_bytes(int E, int R, int C) {
  if (E < 1 || R < 0 || C < 0) return 0;
  return mma_atoms_bytes(E, R, C);
}

