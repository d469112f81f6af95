// permute.cuh -- step 3 of the layer: group the (token, slot) pairs by expert
// and gather the token rows into expert-contiguous order; and the combine
// that forms the layer's output from the expert GEMMs' rows.
//
// The expert-parallel dispatch of the DeepSeek-V3 technical report (section
// 3.2.1, all-to-all dispatch and combine) sends each token to the experts
// chosen for it.  On one GPU the same step is a stable counting sort: expert
// e's tokens land in rows [row_start[e], row_start[e] + counts[e]) in
// ascending token order; row_start pads every expert's segment to a multiple
// of 256 rows so that no GEMM tile straddles two experts.
#pragma once

#include "sm100.cuh"

namespace fgs {

constexpr int kPermThreads = 256;
constexpr int kPermBlockTokens = 128;  // same token blocks as the router

struct PermuteArgs {
  int T, K, N, d, split;
  const int32_t* idx;         // [T, K]
  const float* gate;          // [T, K]
  const int32_t* block_base;  // [nblk, N] first rank of this block's tokens within each expert
  const int32_t* offsets;     // [N + 1] unpadded
  const int32_t* row_start;   // [N + 1] padded
  int32_t* src;               // [T * K] token ids, expert-contiguous (unpadded)
  int32_t* slot_of;           // [T, K] padded row of (t, k)
  float* gate_perm;           // [padded rows] gate of the pair in each row
  const __nv_bfloat16* x;     // [T, d]
  __nv_bfloat16* x_perm;      // [padded rows, d]
  int gather;
  int* tile_ctr;              // [2] zeroed here for the routed gate/up GEMM that follows
};

// grid (nblk, split): CTA (b, s) ranks block b's pairs (cheap, repeated by
// every s) and copies the rows of the tokens tl with tl % split == s.
__global__ void __launch_bounds__(kPermThreads) permute_gather_kernel(PermuteArgs a) {
  __shared__ uint32_t masks[256 * 4];
  __shared__ int32_t base[256], roff[256], rstart[256];
  __shared__ int32_t dst[kPermBlockTokens * 8];
  const int tid = threadIdx.x;
  const int b = blockIdx.x, sp = blockIdx.y;
  const int t0 = b * kPermBlockTokens;
  const int ntok = min(kPermBlockTokens, a.T - t0);
  const int K = a.K;

  pdl_launch_dependents();  // the gate/up kernel may start its shared experts' tiles
  pdl_wait();               // the router's outputs are complete and visible from here
  if (b == 0 && blockIdx.y == 0 && tid < 2) a.tile_ctr[tid] = 0;
  for (int i = tid; i < a.N * 4; i += kPermThreads) masks[i] = 0u;
  for (int e = tid; e < a.N; e += kPermThreads) {
    base[e] = a.block_base[static_cast<size_t>(b) * a.N + e];
    roff[e] = a.offsets[e];
    rstart[e] = a.row_start[e];
  }
  __syncthreads();
  if (tid < ntok) {
    for (int k = 0; k < K; ++k) {
      const int e = a.idx[static_cast<size_t>(t0 + tid) * K + k];
      atomicOr(&masks[e * 4 + (tid >> 5)], 1u << (tid & 31));
    }
  }
  __syncthreads();
  if (tid < ntok) {
    const int t = t0 + tid;
    const int w = tid >> 5;
    const uint32_t below = (1u << (tid & 31)) - 1u;
    for (int k = 0; k < K; ++k) {
      const int e = a.idx[static_cast<size_t>(t) * K + k];
      int rank = __popc(masks[e * 4 + w] & below);
      for (int ww = 0; ww < w; ++ww) rank += __popc(masks[e * 4 + ww]);
      const int pos = base[e] + rank;
      const int prow = rstart[e] + pos;
      dst[tid * K + k] = prow;
      if (sp == 0) {
        a.src[roff[e] + pos] = t;
        a.slot_of[static_cast<size_t>(t) * K + k] = prow;
        a.gate_perm[prow] = a.gate[static_cast<size_t>(t) * K + k];
      }
    }
  }
  if (!a.gather) return;
  __syncthreads();
  // gather: one warp per token row, read once, written K times (16-byte vectors)
  const int warp = tid >> 5, lane = tid & 31, nwarps = kPermThreads / 32;
  const int nvec = a.d >> 3;
  for (int tl = sp + a.split * warp; tl < ntok; tl += a.split * nwarps) {
    const uint4* srow = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t0 + tl) * a.d);
    for (int c = lane; c < nvec; c += 32 * 8) {  // 8 vectors per lane: a 4 KB row per pass
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (c + 32 * u < nvec) v[u] = __ldg(srow + c + 32 * u);
      for (int k = 0; k < K; ++k) {
        uint4* drow = reinterpret_cast<uint4*>(a.x_perm + static_cast<size_t>(dst[tl * K + k]) * a.d);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (c + 32 * u < nvec) drow[c + 32 * u] = v[u];
      }
    }
  }
}

struct CombineArgs {
  int T, K, d;
  const __nv_bfloat16* x;   // [T, d]
  const __nv_bfloat16* ys;  // [T, d] the shared experts' output, or nullptr
  const __nv_bfloat16* y;   // [padded rows, d]: g-scaled routed rows
  const int32_t* slot_of;   // [T, K]
  __nv_bfloat16* out;       // [T, d]
  int add_residual, add_routed;
};

// Step 5, the layer's output: out[t] = x[t] + ys[t] + sum_k y[slot_of[t, k]]
// with the routed rows in ascending k (a fixed order, so the result is
// deterministic), summed in fp32 and rounded once to bf16.  One warp per
// (token, chunk of cols_per_warp columns): every lane issues all of its
// 16-byte loads (x, ys and the K routed rows) for 8 columns before it sums,
// so each warp load reads 512 contiguous bytes of one row.  Large batches
// give a warp a whole row (it loops over the row); small batches split the
// row over warps so that enough loads are in flight.
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a, int cols_per_warp) {
  // no early launch of the next kernel: the next forward's router may start
  // only when this forward has finished with every buffer it shares
  pdl_wait();
  const int chunks = (a.d + cols_per_warp - 1) / cols_per_warp;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= a.T * chunks) return;
  const int t = gw / chunks;
  const int c0 = (gw - t * chunks) * cols_per_warp;
  const int c1 = min(a.d, c0 + cols_per_warp);
  const int K = a.add_routed ? a.K : 0;
  int slots[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) slots[k] = k < K ? a.slot_of[static_cast<size_t>(t) * a.K + k] : 0;
  for (int col = c0 + lane * 8; col < c1; col += 256) {
    uint4 v[10];
    int nv = 0;
    if (a.add_residual) v[nv++] = __ldg(reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * a.d + col));
    if (a.ys) v[nv++] = __ldcg(reinterpret_cast<const uint4*>(a.ys + static_cast<size_t>(t) * a.d + col));
    const int base = nv;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < K) v[base + k] = __ldcg(reinterpret_cast<const uint4*>(a.y + static_cast<size_t>(slots[k]) * a.d + col));
    nv = base + K;
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
    for (int i = 0; i < 10; ++i) {
      if (i < nv) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[2 * j] += bf16lo(w[j]);
          acc[2 * j + 1] += bf16hi(w[j]);
        }
      }
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(a.out + static_cast<size_t>(t) * a.d + col) = o;
  }
}

}  // namespace fgs
