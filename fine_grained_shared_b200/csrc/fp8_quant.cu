// Fine-grained FP8 (E4M3) quantization of GEMM operands with power-of-two scales.
//
// DeepSeek-V3 technical report, section 3.3 "FP8 Training": GEMM inputs in FP8,
// each group of values carrying its own scale (fine-grained scaling), the
// activation scales powers of two.  Appendix B.2 "Discussion About Block-Wise
// Quantization": activations are grouped 1 x 128 along the channels in the
// forward pass, weights in 128 x 128 blocks.
//
// Per group: e = the smallest integer with max|x| <= 448 * 2^e, clamped to
// [-127, 127]; code = E4M3(x * 2^-e), round to nearest even.  Because 2^-e is
// a power of two the product is exact in fp32 wherever E4M3 can tell values
// apart, so the conversion rounds once.  Scales are stored as the biased byte
// e + 127 (UE8M0).
//
// Both kernels stream: each input byte is read once, each output byte written
// once (2 B in, 1 B + 1/128 B out per element), so they are bound by HBM.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fgs_moe.h"
#include "fp8_util.cuh"

namespace {

using fgs::amax8;
using fgs::encode8;
using fgs::pow2_neg;
using fgs::scale_exponent;

constexpr int kGroup = 128;
constexpr int kRowThreads = 256;          // 8 warps, one row at a time each
constexpr int kRowBatch = 8;              // 256-column chunks of a row a lane loads before it converts
constexpr int kBlockThreads = 256;        // one CTA per 128 x 128 block, 8 rows of 8 columns per thread

// x bf16 [rows, cols] -> q [rows, cols], scale [rows, groups].  A warp takes
// whole rows (grid-stride); within a row, 256-column chunks in batches of
// kRowBatch: every lane first loads its 8 columns of each chunk of the batch,
// then converts them.  Lanes 0-15 hold a chunk's first group, lanes 16-31 the
// second.  cols is a multiple of 16, so a lane's 8 columns are either all
// inside the row or all past its end.
__global__ void __launch_bounds__(kRowThreads, 3)
quantize_rows_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int cols,
                     uint8_t* __restrict__ q, uint8_t* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  const int chunks = (cols + 2 * kGroup - 1) / (2 * kGroup);
  const int groups = (cols + kGroup - 1) / kGroup;
  const int64_t nwarps = int64_t(gridDim.x) * (kRowThreads / 32);

  for (int64_t r = int64_t(blockIdx.x) * (kRowThreads / 32) + (threadIdx.x >> 5); r < rows; r += nwarps) {
    const __nv_bfloat16* xr = x + r * cols;
    uint8_t* qr = q + r * cols;
    uint8_t* sr = scale + r * groups;
    for (int c0 = 0; c0 < chunks; c0 += kRowBatch) {
      uint4 v[kRowBatch];
#pragma unroll
      for (int u = 0; u < kRowBatch; ++u) {
        const int col = (c0 + u) * (2 * kGroup) + lane * 8;
        v[u] = make_uint4(0u, 0u, 0u, 0u);
        if (c0 + u < chunks && col < cols) v[u] = __ldg(reinterpret_cast<const uint4*>(xr + col));
      }
#pragma unroll
      for (int u = 0; u < kRowBatch; ++u) {
        if (c0 + u >= chunks) break;                 // the same for every lane of the warp
        const int col = (c0 + u) * (2 * kGroup) + lane * 8;
        float a = amax8(v[u]);                       // 0 for lanes past the row's end
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
        const int e = scale_exponent(a);
        if (col < cols) {
          *reinterpret_cast<uint2*>(qr + col) = encode8(v[u], pow2_neg(e));
          if ((lane & 15) == 0) sr[(c0 + u) * 2 + (lane >> 4)] = uint8_t(e + 127);
        }
      }
    }
  }
}

// w bf16 [batch, rows, cols] -> q, scale [batch, ceil(rows/128), ceil(cols/128)].
// CTA (bx, by, bz) = block (by, bx) of matrix bz; thread t covers columns
// 8*(t % 16) .. +8 of rows t/16 + 16 k, k = 0..7.
__global__ void __launch_bounds__(kBlockThreads)
quantize_blocks_kernel(const __nv_bfloat16* __restrict__ w, int rows, int cols,
                       uint8_t* __restrict__ q, uint8_t* __restrict__ scale) {
  __shared__ float warp_max[kBlockThreads / 32];
  const int col = blockIdx.x * kGroup + (threadIdx.x & 15) * 8;
  const int row0 = blockIdx.y * kGroup + (threadIdx.x >> 4);
  const int64_t base = int64_t(blockIdx.z) * rows * cols;

  uint4 v[8];
  float a = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int r = row0 + 16 * k;
    v[k] = make_uint4(0u, 0u, 0u, 0u);
    if (r < rows && col < cols) v[k] = __ldg(reinterpret_cast<const uint4*>(w + base + int64_t(r) * cols + col));
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) a = fmaxf(a, amax8(v[k]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = a;
  __syncthreads();
  a = warp_max[0];
#pragma unroll
  for (int i = 1; i < kBlockThreads / 32; ++i) a = fmaxf(a, warp_max[i]);
  const int e = scale_exponent(a);
  const float inv = pow2_neg(e);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int r = row0 + 16 * k;
    if (r < rows && col < cols)
      *reinterpret_cast<uint2*>(q + base + int64_t(r) * cols + col) = encode8(v[k], inv);
  }
  if (threadIdx.x == 0) {
    const int gr = (rows + kGroup - 1) / kGroup, gc = (cols + kGroup - 1) / kGroup;
    scale[(int64_t(blockIdx.z) * gr + blockIdx.y) * gc + blockIdx.x] = uint8_t(e + 127);
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

}  // namespace

extern "C" moe_status moe_quantize_fp8_rows(const void* x, int64_t rows, int32_t cols, uint8_t* q,
                                            uint8_t* scale, void* stream) {
  if (!x || !q || !scale) return MOE_ERR_INVALID_ARG;
  if (rows < 0 || cols <= 0) return MOE_ERR_SHAPE;
  if (cols % 16 != 0 || !aligned16(x) || !aligned16(q)) return MOE_ERR_ALIGNMENT;
  if (rows == 0) return MOE_OK;
  const int sms = sm_count();
  if (sms <= 0) return MOE_ERR_CUDA;
  const int64_t per_block = kRowThreads / 32;
  int64_t blocks = (rows + per_block - 1) / per_block;
  int per_sm = 0;  // one wave of the grid-stride loop: the CTAs that fit on the GPU at once
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_rows_kernel, kRowThreads, 0) != cudaSuccess ||
      per_sm <= 0)
    return MOE_ERR_CUDA;
  const int64_t resident = int64_t(sms) * per_sm;
  if (blocks > resident) blocks = resident;
  quantize_rows_kernel<<<unsigned(blocks), kRowThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), rows, cols, q, scale);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" moe_status moe_quantize_fp8_blocks(const void* w, int32_t batch, int32_t rows, int32_t cols,
                                              uint8_t* q, uint8_t* scale, void* stream) {
  if (!w || !q || !scale) return MOE_ERR_INVALID_ARG;
  if (batch < 0 || rows < 0 || cols <= 0 || batch > 65535 || (int64_t(rows) + kGroup - 1) / kGroup > 65535)
    return MOE_ERR_SHAPE;
  if (cols % 16 != 0 || !aligned16(w) || !aligned16(q)) return MOE_ERR_ALIGNMENT;
  if (batch == 0 || rows == 0) return MOE_OK;
  const dim3 grid(unsigned((cols + kGroup - 1) / kGroup), unsigned((rows + kGroup - 1) / kGroup), unsigned(batch));
  quantize_blocks_kernel<<<grid, kBlockThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(w), rows, cols, q, scale);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
