// ep.cuh -- the steps an expert-parallel layer adds to the single-GPU forward
// (DeepSeek-V3 technical report summary, section 3.2.1: all-to-all dispatch of
// the tokens to the experts' ranks and combine of the results), written as
// kernels that address the other ranks' workspaces directly (peer loads and
// stores over NVLink; on one GPU, the same kernels over several handles'
// workspaces):
//
//   ep_plan_kernel      every rank's per-expert counts -> this rank's destination
//                       rows (ep_plan.h) and its own experts' GEMM tables
//   ep_dispatch_kernel  the permutation of permute.cuh with each (token, slot)
//                       row, and its gate, stored into the buffer of the rank
//                       that holds the slot's expert; in the FP8 layer the row
//                       is quantized once (1 x 128 groups, as permute_quant_kernel)
//                       and its E4M3 codes and scale cells are what is sent
//                       (the DeepSeek-V3 report's FP8 dispatch, section 3.3)
//   ep_combine_kernel   out[t] = x[t] + ys[t] + sum_k y_owner(k)[slot_of[t, k]],
//                       the g-scaled rows loaded from their owners, k ascending
//
// The ranks order these steps by stream-ordered barriers between them (one
// small all-reduce each): counts before the plan, rows before the GEMMs, the
// GEMMs' rows before the combine.  No step waits on another rank inside a
// kernel, and no load of another rank's memory is a TMA load: the owner's GEMMs
// read only their own workspace.
#pragma once

#include "ep_plan.h"
#include "fp8_gemm.cuh"
#include "permute.cuh"

namespace fgs {

// every rank's workspace base as this device addresses it (this rank's own included)
struct EpPeers {
  uint8_t* ws[kEpMaxRanks];
};

struct EpPlanArgs {
  int G, N, rank;
  size_t counts_off;         // byte offset of the router's counts [N] in every workspace
  EpPeers peers;
  int32_t* base;             // [N] first row of this rank's rows of expert e in the buffer of e's rank
  int32_t* counts_loc;       // [N / G + 1] rows of each local expert over all ranks
  int32_t* row_start;        // [N / G + 1]
  int32_t* mtile_start;      // [N / G + 1] prefix of ceil(rows / 256)
  int32_t* mtile128_start;   // [N / G + 1] prefix of ceil(rows / 128)
};

constexpr int kEpPlanThreads = 256;

__host__ __device__ constexpr size_t ep_plan_smem_bytes(int G, int N) {
  return static_cast<size_t>(G) * static_cast<size_t>(N) * 4;
}

// one CTA: all ranks' counts into shared memory, then the plan's entries, one thread each
__global__ void __launch_bounds__(kEpPlanThreads) ep_plan_kernel(EpPlanArgs a) {
  extern __shared__ int32_t s_cnt[];  // [G][N]
  const int tid = threadIdx.x;
  for (int i = tid; i < a.G * a.N; i += kEpPlanThreads) {
    const int r = i / a.N, e = i - r * a.N;
    s_cnt[i] = __ldcg(reinterpret_cast<const int32_t*>(a.peers.ws[r] + a.counts_off) + e);
  }
  __syncthreads();
  const int32_t* rows[kEpMaxRanks];
  for (int r = 0; r < a.G; ++r) rows[r] = s_cnt + r * a.N;
  for (int e = tid; e < a.N; e += kEpPlanThreads) a.base[e] = ep_dest_base(rows, a.G, a.N, a.rank, e);
  const int per = a.N / a.G;
  for (int l = tid; l <= per; l += kEpPlanThreads) {
    int32_t c, rs, mt, m128;
    ep_owner_entry(rows, a.G, a.N, a.rank, l, &c, &rs, &mt, &m128);
    a.counts_loc[l] = c;
    a.row_start[l] = rs;
    a.mtile_start[l] = mt;
    a.mtile128_start[l] = m128;
  }
}

struct EpDispatchArgs {
  int T, K, N, d, split, per_rank;
  const int32_t* idx;         // [T, K] global expert ids
  const float* gate;          // [T, K]
  const int32_t* block_base;  // [nblk, N] first rank of this block's tokens within each expert (router)
  const int32_t* offsets;     // [N + 1] this rank's unpadded offsets (for src)
  const int32_t* base;        // [N] from ep_plan_kernel
  int32_t* src;               // [T * K] this rank's tokens, expert-contiguous
  int32_t* slot_of;           // [T, K] row of (t, k) in the buffer of its expert's rank
  const __nv_bfloat16* x;     // [T, d]
  size_t xperm_off, gate_off;  // byte offsets of the row buffer and its gates in every workspace
  EpPeers peers;
  int* tile_ctr;              // [2] this rank's gate/up tile counter, zeroed for its GEMMs
  // FP8 layer: byte offsets of the codes [P, d] and scale atoms of the row buffer in every
  // workspace, and this rank's own dense codes of x with their atoms (the shared experts' A) or null
  size_t xq_off, xs_off;
  uint8_t* xq;
  uint8_t* xs;
};

// grid (nblk, split), as permute_gather_kernel: CTA (b, s) ranks block b's
// pairs and copies the rows of the tokens tl with tl % split == s to every
// rank that holds one of the token's experts (one 16-byte store stream per
// (token, slot) pair; a rank that holds several of a token's experts receives
// the row once per expert, the layout its grouped GEMMs read).
template <bool FP8>
__global__ void __launch_bounds__(kPermThreads) ep_dispatch_kernel(EpDispatchArgs a) {
  __shared__ uint32_t masks[256 * 4];
  __shared__ int32_t sbase[256], roff[256], ebase[256];
  __shared__ int32_t dst[kPermBlockTokens * 8];
  __shared__ uint8_t dstq[kPermBlockTokens * 8];
  const int tid = threadIdx.x;
  const int b = blockIdx.x, sp = blockIdx.y;
  const int t0 = b * kPermBlockTokens;
  const int ntok = min(kPermBlockTokens, a.T - t0);
  const int K = a.K;
  if (b == 0 && sp == 0 && tid < 2) a.tile_ctr[tid] = 0;
  for (int i = tid; i < a.N * 4; i += kPermThreads) masks[i] = 0u;
  for (int e = tid; e < a.N; e += kPermThreads) {
    sbase[e] = a.block_base[static_cast<size_t>(b) * a.N + e];
    roff[e] = a.offsets[e];
    ebase[e] = a.base[e];
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
      const int pos = sbase[e] + rank;
      const int prow = ebase[e] + pos;
      const int q = e / a.per_rank;
      dst[tid * K + k] = prow;
      dstq[tid * K + k] = static_cast<uint8_t>(q);
      if (sp == 0) {
        a.src[roff[e] + pos] = t;
        a.slot_of[static_cast<size_t>(t) * K + k] = prow;
        reinterpret_cast<float*>(a.peers.ws[q] + a.gate_off)[prow] = a.gate[static_cast<size_t>(t) * K + k];
      }
    }
  }
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31, nwarps = kPermThreads / 32;
  if constexpr (FP8) {
    // quantize each token row once: a warp per row, 256 columns (two 128-column groups) per pass,
    // lanes 0-15 the first group and 16-31 the second; codes and scale cells to every destination
    const int groups = a.d / kF8BK;
    for (int tl = sp + a.split * warp; tl < ntok; tl += a.split * nwarps) {
      const size_t t = static_cast<size_t>(t0 + tl);
      const __nv_bfloat16* srow = a.x + t * a.d;
      for (int c0 = 0; c0 < a.d; c0 += 2 * kF8BK) {
        const int col = c0 + lane * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (col < a.d) v = __ldg(reinterpret_cast<const uint4*>(srow + col));
        float m = amax8(v);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const int e = scale_exponent(m);
        if (col < a.d) {
          const uint2 codes = encode8(v, pow2_neg(e));
          const int g = col / kF8BK;
          const uint32_t sbyte = static_cast<uint32_t>(e + 127);
          for (int k = 0; k < K; ++k) {
            uint8_t* ws = a.peers.ws[dstq[tl * K + k]];
            const size_t R = static_cast<size_t>(dst[tl * K + k]);
            *reinterpret_cast<uint2*>(ws + a.xq_off + R * a.d + col) = codes;
            if ((lane & 15) == 0) put_scale(ws + a.xs_off, R, g, groups, sbyte);
          }
          if (a.xq) {
            *reinterpret_cast<uint2*>(a.xq + t * a.d + col) = codes;
            if ((lane & 15) == 0) put_scale(a.xs, t, g, groups, sbyte);
          }
        }
      }
    }
    __threadfence_system();
    return;
  }
  // one warp per token row, read once and stored to each of its K destinations
  const int nvec = a.d >> 3;
  for (int tl = sp + a.split * warp; tl < ntok; tl += a.split * nwarps) {
    const uint4* srow = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t0 + tl) * a.d);
    for (int c = lane; c < nvec; c += 32 * 8) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (c + 32 * u < nvec) v[u] = __ldg(srow + c + 32 * u);
      for (int k = 0; k < K; ++k) {
        uint4* drow = reinterpret_cast<uint4*>(a.peers.ws[dstq[tl * K + k]] + a.xperm_off) +
                      static_cast<size_t>(dst[tl * K + k]) * nvec;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (c + 32 * u < nvec) drow[c + 32 * u] = v[u];
      }
    }
  }
  // the rows and gates are in the other ranks' memory before the barrier that follows this kernel
  __threadfence_system();
}

struct EpCombineArgs {
  int T, K, d, per_rank;
  const __nv_bfloat16* x;   // [T, d]
  const __nv_bfloat16* ys;  // [T, d] this rank's shared experts' output, or nullptr
  const int32_t* idx;       // [T, K]
  const int32_t* slot_of;   // [T, K] row in the buffer of the slot's expert's rank
  size_t y_off;             // byte offset of the g-scaled routed rows in every workspace
  EpPeers peers;
  __nv_bfloat16* out;       // [T, d]
  int add_residual, add_routed;
};

// combine_kernel's sum with each routed row loaded from the rank that computed
// it: one warp per (token, chunk of cols_per_warp columns), all 16-byte loads of
// a lane's 8 columns issued before the sum, fp32 sum in ascending k, one bf16
// rounding.
__global__ void __launch_bounds__(256) ep_combine_kernel(EpCombineArgs a, int cols_per_warp) {
  const int chunks = (a.d + cols_per_warp - 1) / cols_per_warp;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= a.T * chunks) return;
  const int t = gw / chunks;
  const int c0 = (gw - t * chunks) * cols_per_warp;
  const int c1 = min(a.d, c0 + cols_per_warp);
  const int K = a.add_routed ? a.K : 0;
  const __nv_bfloat16* yrow[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    yrow[k] = a.x;
    if (k < K) {
      const size_t i = static_cast<size_t>(t) * a.K + k;
      const int q = a.idx[i] / a.per_rank;
      yrow[k] = reinterpret_cast<const __nv_bfloat16*>(a.peers.ws[q] + a.y_off) +
                static_cast<size_t>(a.slot_of[i]) * a.d;
    }
  }
  auto add8 = [](float (&acc)[8], const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      acc[2 * j] += bf16lo(w[j]);
      acc[2 * j + 1] += bf16hi(w[j]);
    }
  };
  for (int col = c0 + lane * 8; col < c1; col += 256) {
    const size_t xo = static_cast<size_t>(t) * a.d + col;
    uint4 vx = make_uint4(0u, 0u, 0u, 0u), vs = vx, vy[8];
    if (a.add_residual) vx = __ldg(reinterpret_cast<const uint4*>(a.x + xo));
    if (a.ys) vs = __ldcg(reinterpret_cast<const uint4*>(a.ys + xo));
#pragma unroll
    for (int k = 0; k < 8; ++k) vy[k] = k < K ? __ldcg(reinterpret_cast<const uint4*>(yrow[k] + col)) : vx;
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    if (a.add_residual) add8(acc, vx);
    if (a.ys) add8(acc, vs);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < K) add8(acc, vy[k]);
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(a.out + xo) = o;
  }
}

}  // namespace fgs
