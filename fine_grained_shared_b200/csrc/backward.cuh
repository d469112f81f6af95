// backward.cuh -- the streaming and CUDA-core steps of the layer's backward
// pass: input, router and expert-weight gradients (DeepSeek-V3 technical report summary,
// section 3.2.1 "DualPipe and Computation-Communication Overlap": the MoE
// layer's backward for input and backward for weights are separate pieces of
// a training step; the formulas are the chain rule through the forward).
//
// With dh the gradient of the layer output, for a routed row (token t, slot k,
// expert e, gate g) and m = SiLU(a) * b, a = W_gate x, b = W_up x:
//   dm_raw = W_down^T dh               (grouped GEMM, down_gemm.cuh)
//   dg     = dm_raw . m                (partial sums in the recompute's epilogue)
//   da, db = g dm_raw b SiLU'(a), g dm_raw SiLU(a)   (gateup_gemm_kernel<true>)
//   dx_row = W_gate^T da + W_up^T db   (grouped GEMM, down_gemm.cuh)
//   dx[t]  = dh[t] + shared rows' dx + sum_k dx_row(t, k) + (dz E)[t]
// and through the gates to the router logits z (softmax: dz = s (ds - s.ds),
// ds_i = the dg of the slot that chose i; sigmoid, g = s / S over the chosen:
// ds_k = (dg_k - g . dg) / S, dz = ds s (1 - s) on the chosen experts):
//   dE = dz^T x, d(logit bias) = sum_t dz.
// This file holds the steps that are not tensor-core GEMMs: the weight
// transposes that give the data-gradient GEMMs K-major operands, the gather of
// dh into the expert-ordered rows (and g dh for the weight gradients), the gate
// gradient's reduction, the router's dz step (the softmax or sigmoid Jacobian
// per token; its three contractions run on the tensor cores) and the final sum.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace fgs {

// ---------------------------------------------------------------------------
// Transposes through shared memory, tiles of 64 x 64: each thread loads 32
// contiguous bytes of one source row and stores 32 contiguous bytes (16
// source rows) of one destination row.
// ---------------------------------------------------------------------------
constexpr int kTrRows = 64, kTrCols = 64;

// tile[r][c] <- src rows r0 .. + 63 (rows >= nrows zero), columns c0 .. + 63 (C a multiple of 16)
__device__ __forceinline__ void tr_load_tile(uint16_t (*tile)[kTrCols + 2], const uint16_t* src, long long ld, int C,
                                             int r0, int nrows, int c0) {
  const int tr = threadIdx.x >> 2, tc = (threadIdx.x & 3) * 16;
  uint4 v0 = make_uint4(0u, 0u, 0u, 0u), v1 = v0;
  if (r0 + tr < nrows && c0 + tc < C) {
    const uint4* p = reinterpret_cast<const uint4*>(src + static_cast<size_t>(r0 + tr) * ld + c0 + tc);
    v0 = p[0];
    v1 = p[1];
  }
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    tile[tr][tc + 2 * j] = static_cast<uint16_t>(w[j] & 0xFFFFu);
    tile[tr][tc + 2 * j + 1] = static_cast<uint16_t>(w[j] >> 16);
  }
}

// dst row (c0 + oc), values of source rows r0 + orr .. + 15: thread (oc = tid / 4, orr = (tid % 4) * 16)
__device__ __forceinline__ void tr_store_row(const uint16_t (*tile)[kTrCols + 2], uint16_t* q, int nvalid, int orr,
                                             int oc) {
  uint32_t w[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t lo = tile[orr + 2 * j][oc], hi = tile[orr + 2 * j + 1][oc];
    w[j] = lo | (hi << 16);
  }
  if (nvalid >= 16 && (reinterpret_cast<uintptr_t>(q) & 15u) == 0) {
    reinterpret_cast<uint4*>(q)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(q)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < nvalid) q[j] = static_cast<uint16_t>(w[j >> 1] >> ((j & 1) * 16));
  }
}

// ---------------------------------------------------------------------------
// Batched transpose: dst[b][c][col0 + r] = src[b][r][c], r < R, c < C (R, C,
// dst_ld and col0 multiples of 16).
// ---------------------------------------------------------------------------
struct TransposeArgs {
  const __nv_bfloat16* src;
  __nv_bfloat16* dst;
  int R, C, dst_ld, col0;
  long long src_bs, dst_bs;  // batch strides in elements
};

__global__ void __launch_bounds__(256) transpose_bf16_kernel(TransposeArgs a) {
  __shared__ uint16_t tile[kTrRows][kTrCols + 2];
  const int c0 = blockIdx.x * kTrCols, r0 = blockIdx.y * kTrRows, b = blockIdx.z;
  const uint16_t* src = reinterpret_cast<const uint16_t*>(a.src) + b * a.src_bs;
  uint16_t* dst = reinterpret_cast<uint16_t*>(a.dst) + b * a.dst_bs;
  tr_load_tile(tile, src, a.C, a.C, r0, a.R, c0);
  __syncthreads();
  const int oc = threadIdx.x >> 2, orr = (threadIdx.x & 3) * 16;
  if (c0 + oc >= a.C || r0 + orr >= a.R) return;
  tr_store_row(tile, dst + static_cast<size_t>(c0 + oc) * a.dst_ld + a.col0 + r0 + orr, a.R - r0 - orr, orr, oc);
}

// ---------------------------------------------------------------------------
// Zero, in each expert's segment, the rows past its count up to the next
// multiple of 64 rows, in a [rows, d] and (if given) b [rows, d]: the
// weight-gradient GEMMs sum over whole 64-row blocks of an expert's rows, and a
// padding row may still hold an earlier call's values, which a zero operand
// on the other side would not cancel if they are not finite.  One CTA per
// expert; d a multiple of 8.  The rows stay inside the segment, which is
// padded to a multiple of 256 rows.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) zero_tail_rows_kernel(const int32_t* row_start, const int32_t* counts, int d,
                                                             __nv_bfloat16* a, __nv_bfloat16* b) {
  const int e = blockIdx.x;
  const int cnt = counts[e];
  const int n = ((cnt + 63) & ~63) - cnt;  // rows to clear, 0 .. 63
  const size_t r0 = static_cast<size_t>(row_start[e]) + static_cast<size_t>(cnt);
  const int per_row = d >> 3;              // 16-byte units per row
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (int i = threadIdx.x; i < n * per_row; i += blockDim.x) {
    const int r = i / per_row, c = i - r * per_row;
    const size_t off = (r0 + static_cast<size_t>(r)) * static_cast<size_t>(d) + static_cast<size_t>(c) * 8;
    *reinterpret_cast<uint4*>(a + off) = z;
    if (b) *reinterpret_cast<uint4*>(b + off) = z;
  }
}

// the shared experts' K ranges for the weight-gradient GEMMs: every expert j < n over rows [0, T)
__global__ void fill_dense_groups_kernel(int32_t* k_start, int32_t* k_count, int n, int T) {
  const int i = threadIdx.x;
  if (i < n) {
    k_start[i] = 0;
    k_count[i] = T;
  }
}

// ---------------------------------------------------------------------------
// dh into the expert-ordered rows: dh_perm[slot[t, k]] = dh[t], and (dy not null)
// dy[slot[t, k]] = g[t, k] dh[t], the weight gradient's operand; a warp per (t, k)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_gather_kernel(const __nv_bfloat16* __restrict__ dh, const int32_t* slot_of,
                                                        int TK, int K, int d, __nv_bfloat16* dh_perm,
                                                        const float* gate, __nv_bfloat16* dy) {
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (w >= TK) return;
  const int t = w / K;
  const size_t row = static_cast<size_t>(slot_of[w]);
  const uint4* s = reinterpret_cast<const uint4*>(dh + static_cast<size_t>(t) * d);
  uint4* o = reinterpret_cast<uint4*>(dh_perm + row * d);
  uint4* oy = dy ? reinterpret_cast<uint4*>(dy + row * d) : nullptr;
  const float g = dy ? gate[w] : 0.f;
  for (int c = lane; c < (d >> 3); c += 32) {
    const uint4 v = __ldg(s + c);
    o[c] = v;
    if (oy) {
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
      uint32_t q[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) q[j] = pack_bf16x2(g * bf16lo(wv[j]), g * bf16hi(wv[j]));
      oy[c] = make_uint4(q[0], q[1], q[2], q[3]);
    }
  }
}

// ---------------------------------------------------------------------------
// dgate[t, k] = sum over the 128-column tiles n (ascending) of dg_part[slot[t, k], n]
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dg_reduce_kernel(const float* dg_part, const int32_t* slot_of, int TK,
                                                       int n_tiles, float* dgate) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= TK) return;
  const float* p = dg_part + static_cast<size_t>(slot_of[i]) * n_tiles;
  float s = 0.f;
  for (int n = 0; n < n_tiles; ++n) s += p[n];
  dgate[i] = s;
}

// ---------------------------------------------------------------------------
// The router's backward between its three GEMMs (z = x E^T, dz E and dz^T x,
// on the tensor cores): per token, the affinities from the recomputed logits
// z (+ c) and dz from the gates' gradient; a warp per token.  Writes dz in
// fp32 [T, N] (for d(logit bias)) and in bf16 [T, Npad] (the GEMMs' operand,
// zero in the padding columns).
// ---------------------------------------------------------------------------
struct RouterDzArgs {
  int T, N, Npad, K, sigmoid;
  const float* z;            // [T, Npad] logits x E^T (without the logit bias)
  const float* logit_bias;   // [N] or nullptr (softmax)
  const int32_t* idx;        // [T, K]
  const float* dgate;        // [T, K]
  float* dz;                 // [T, N] out
  __nv_bfloat16* dzb;        // [T, Npad] out
};

__global__ void __launch_bounds__(256) router_dz_kernel(RouterDzArgs a) {
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (t >= a.T) return;
  const int N = a.N, K = a.K;
  const float* zr = a.z + static_cast<size_t>(t) * a.Npad;
  float zv[8];  // experts lane + 32 j
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = lane + 32 * j;
    zv[j] = i < N ? zr[i] + (a.logit_bias ? a.logit_bias[i] : 0.f) : -INFINITY;
  }
  int ki[8];
  float kg[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    ki[k] = k < K ? a.idx[static_cast<size_t>(t) * K + k] : -1;
    kg[k] = k < K ? a.dgate[static_cast<size_t>(t) * K + k] : 0.f;
  }
  float dzv[8];
  if (!a.sigmoid) {
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) mx = fmaxf(mx, zv[j]);
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sv[8], sum = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      sv[j] = lane + 32 * j < N ? __expf(zv[j] - mx) : 0.f;
      sum += sv[j];
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = 1.f / sum;
    // s . ds = sum over the chosen slots of s_i dg_k (each chosen expert once)
    float sds = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = lane + 32 * j;
      sv[j] *= inv;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (ki[k] == i) sds += sv[j] * kg[k];
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) sds += __shfl_xor_sync(0xffffffffu, sds, o);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = lane + 32 * j;
      float ds = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (ki[k] == i) ds = kg[k];
      dzv[j] = sv[j] * (ds - sds);
    }
  } else {
    // g_k = s_k / S over the chosen; ds_k = (dg_k - g . dg) / S; dz = ds s (1 - s) there, 0 elsewhere
    float S = 0.f, sdg = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = lane + 32 * j;
      const float s = 1.f / (1.f + __expf(-zv[j]));
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (ki[k] == i) {
          S += s;
          sdg += s * kg[k];
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      S += __shfl_xor_sync(0xffffffffu, S, o);
      sdg += __shfl_xor_sync(0xffffffffu, sdg, o);
    }
    const float gdg = sdg / S;  // sum over the chosen of g_l dg_l
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = lane + 32 * j;
      const float s = 1.f / (1.f + __expf(-zv[j]));
      float v = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (ki[k] == i) v = (kg[k] - gdg) / S * s * (1.f - s);
      dzv[j] = v;
    }
  }
  float* dzr = a.dz + static_cast<size_t>(t) * N;
  __nv_bfloat16* dbr = a.dzb + static_cast<size_t>(t) * a.Npad;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = lane + 32 * j;
    if (i < N) dzr[i] = dzv[j];
    if (i < a.Npad) dbr[i] = __float2bfloat16_rn(i < N ? dzv[j] : 0.f);
  }
}

// d(logit bias)_i = sum over t (ascending) of dz[t, i]; a thread per expert
__global__ void __launch_bounds__(256) column_sum_kernel(const float* dz, int T, int N, float* out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  float s = 0.f;
  for (int t = 0; t < T; ++t) s += dz[static_cast<size_t>(t) * N + i];
  out[i] = s;
}

// the K ranges of a GEMM split into `n` segments of `seg` rows (the last one shorter) over [0, total)
__global__ void fill_segments_kernel(int32_t* k_start, int32_t* k_count, int n, int seg, int total) {
  const int i = threadIdx.x;
  if (i < n) {
    k_start[i] = i * seg;
    k_count[i] = min(seg, total - i * seg);
  }
}

__global__ void __launch_bounds__(256) router_de_reduce_kernel(const float* part, int segments, size_t n,
                                                              float* out) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float s = 0.f;
  for (int g = 0; g < segments; ++g) s += part[static_cast<size_t>(g) * n + i];
  out[i] = s;
}

// ---------------------------------------------------------------------------
// dx[t] = dh[t] + dxs[t] + dx_router[t] + sum_k dx_perm[slot[t, k]] (k ascending), fp32, one rounding;
// a warp per (token, chunk of cols_per_warp columns)
// ---------------------------------------------------------------------------
struct BwdCombineArgs {
  int T, K, d;
  const __nv_bfloat16* dh;       // or nullptr (no residual)
  const __nv_bfloat16* dxs;      // shared experts' rows, or nullptr
  const float* dx_router;        // or nullptr
  const __nv_bfloat16* dx_perm;  // routed rows, or nullptr
  const int32_t* slot_of;
  __nv_bfloat16* dx;
};

__global__ void __launch_bounds__(256) bwd_combine_kernel(BwdCombineArgs a, int cols_per_warp) {
  const int chunks = (a.d + cols_per_warp - 1) / cols_per_warp;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (gw >= a.T * chunks) return;
  const int t = gw / chunks;
  const int c0 = (gw - t * chunks) * cols_per_warp, c1 = min(a.d, c0 + cols_per_warp);
  const int K = a.dx_perm ? a.K : 0;
  int slots[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) slots[k] = k < K ? a.slot_of[static_cast<size_t>(t) * a.K + k] : 0;
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
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    if (a.dh) add8(acc, __ldg(reinterpret_cast<const uint4*>(a.dh + xo)));
    if (a.dxs) add8(acc, __ldcg(reinterpret_cast<const uint4*>(a.dxs + xo)));
    if (a.dx_router) {
      const float4 r0 = __ldcg(reinterpret_cast<const float4*>(a.dx_router + xo));
      const float4 r1 = __ldcg(reinterpret_cast<const float4*>(a.dx_router + xo) + 1);
      acc[0] += r0.x; acc[1] += r0.y; acc[2] += r0.z; acc[3] += r0.w;
      acc[4] += r1.x; acc[5] += r1.y; acc[6] += r1.z; acc[7] += r1.w;
    }
    uint4 vy[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      vy[k] = k < K ? __ldcg(reinterpret_cast<const uint4*>(a.dx_perm + static_cast<size_t>(slots[k]) * a.d + col))
                    : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < K) add8(acc, vy[k]);
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(a.dx + xo) = o;
  }
}

}  // namespace fgs
