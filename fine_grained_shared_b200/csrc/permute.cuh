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

#include "router_topk.cuh"
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

// ---------------------------------------------------------------------------
// Steps 1-3 for a decode batch with a small router matrix (T <= 128 tokens,
// N <= 256 experts, N * d * 2 <= 1 MB) in one launch, built around the
// latency of its few dependent steps rather than bandwidth.  One cluster of
// kRouteCluster CTAs per token: warp w of CTA r computes the logits of experts
// i with i % 64 == 8 r + w (two at a time, each lane summing its columns
// c = lane + 32 j in the same order as router_small_kernel, so the logits are
// the same bit for bit) and stores them into the shared memory of the
// cluster's CTA 0, which, after a cluster barrier, selects the token's K
// experts: thread i ranks expert i against the others by (key descending,
// index ascending) -- the order of router_small_kernel's argmax rounds --
// instead of K rounds of warp shuffles.  The cluster whose token is counted
// last (one global counter) then forms the tables and the permutation of the
// whole batch with all of its CTAs: each reads every token's choices, counts
// and scans them (one warp, shuffle scans), and ranks the pairs; CTA 0 writes
// the tables, and the CTAs' warps copy the pairs' rows.
// On the 16B decode layer (T = 32) the router's cross-CTA steps and the
// separate permutation had kept the routed experts' rows from the gate/up
// GEMM until 16 us into the forward.
// ---------------------------------------------------------------------------
constexpr int kRouteCluster = 8;
constexpr int kRouteThreads = 256;
constexpr int kRouteMaxT = 128;
constexpr size_t kRouteMaxRouterBytes = size_t(1) << 20;

__host__ __device__ constexpr bool route_decode_fits(long long T, long long N, long long d, long long K) {
  return T >= 1 && T <= kRouteMaxT && N <= 256 && K <= 8 &&
         static_cast<size_t>(N) * static_cast<size_t>(d) * 2 <= kRouteMaxRouterBytes;
}

struct RouteTables {
  int32_t* counts;          // [N]
  int32_t* offsets;         // [N + 1] unpadded
  int32_t* row_start;       // [N + 1] padded to kExpertRowAlign
  int32_t* mtile_start;     // [N + 1] prefix sum of ceil(count / kExpertRowAlign)
  int32_t* mtile128_start;  // [N + 1] prefix sum of ceil(count / 128)
  int32_t* block_counts;    // [1, N] the one block's exclusive bases (zeros)
};

template <bool SIGMOID>
__global__ void __cluster_dims__(kRouteCluster, 1, 1) __launch_bounds__(kRouteThreads)
    route_permute_decode_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ e,
                                RouterArgs a, PermuteArgs p, RouteTables rt) {
  __shared__ float z[256], key[256], sval[256];
  __shared__ int sel[8];
  __shared__ uint32_t allowed_s, is_last;
  __shared__ uint32_t masks[256 * 4];
  __shared__ int32_t cnt[256], roff[257], rstart[257], mt[257], mt128[257];
  __shared__ int32_t dst[kRouteMaxT * 8];
  const int r = static_cast<int>(cluster_ctarank());
  const int t = blockIdx.x / kRouteCluster;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d = p.d, K = p.K, N = a.N, T = a.T;
  pdl_wait();
  pdl_launch_dependents();
  // CTA 0's bias loads go out first; they are used after the logits
  const float* gb = SIGMOID ? a.select_bias : a.logit_bias;
  const float bias = (r == 0 && gb && tid < N) ? __ldg(gb + tid) : 0.f;
  // ---- logits of this CTA's experts, into CTA 0's z ----
  {
    const int nvec = d >> 3;
    const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d);
    const uint32_t z0 = mapa_shared(smem_u32(z), 0);
    for (int i0 = r * 8 + warp; i0 < N; i0 += 2 * 8 * kRouteCluster) {
      const int i1 = i0 + 8 * kRouteCluster;
      const bool two = i1 < N;
      const uint4* er0 = reinterpret_cast<const uint4*>(e + static_cast<size_t>(i0) * d);
      const uint4* er1 = reinterpret_cast<const uint4*>(e + static_cast<size_t>(two ? i1 : i0) * d);
      float acc0 = 0.f, acc1 = 0.f;
      for (int c0 = 0; c0 < nvec; c0 += 32 * kSmallRouterPass) {
        uint4 xv[kSmallRouterPass], ev0[kSmallRouterPass], ev1[kSmallRouterPass];
#pragma unroll
        for (int j = 0; j < kSmallRouterPass; ++j) {
          const int c = c0 + lane + 32 * j;
          const int cc = c < nvec ? c : 0;
          xv[j] = ldg_v4_ordered(xr + cc);
          ev0[j] = ldg_v4_ordered(er0 + cc);
        }
        if (two) {
#pragma unroll
          for (int j = 0; j < kSmallRouterPass; ++j) {
            const int c = c0 + lane + 32 * j;
            ev1[j] = ldg_v4_ordered(er1 + (c < nvec ? c : 0));
          }
        } else {
#pragma unroll
          for (int j = 0; j < kSmallRouterPass; ++j) ev1[j] = make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int j = 0; j < kSmallRouterPass; ++j) {
          if (c0 + lane + 32 * j < nvec) {
            const uint32_t xw[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
            const uint32_t w0[4] = {ev0[j].x, ev0[j].y, ev0[j].z, ev0[j].w};
            const uint32_t w1[4] = {ev1[j].x, ev1[j].y, ev1[j].z, ev1[j].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              acc0 = fmaf(bf16lo(xw[q]), bf16lo(w0[q]), acc0);
              acc0 = fmaf(bf16hi(xw[q]), bf16hi(w0[q]), acc0);
              acc1 = fmaf(bf16lo(xw[q]), bf16lo(w1[q]), acc1);
              acc1 = fmaf(bf16hi(xw[q]), bf16hi(w1[q]), acc1);
            }
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        acc0 += __shfl_xor_sync(0xffffffffu, acc0, o);
        acc1 += __shfl_xor_sync(0xffffffffu, acc1, o);
      }
      if (lane == 0) {
        st_cluster_f32(z0 + 4u * i0, acc0);
        if (two) st_cluster_f32(z0 + 4u * i1, acc1);
      }
    }
  }
  cluster_sync();  // CTA 0 holds all N logits
  // ---- CTA 0: the token's selection ----
  if (r == 0) {
    if (tid < N) {
      const float zi = z[tid];
      float k;
      if (SIGMOID) {
        const float sv = 1.f / (1.f + __expf(-zi));
        sval[tid] = sv;
        k = sv + bias;
      } else {
        k = zi + bias;  // softmax is monotone in z
      }
      key[tid] = isnan(k) ? -INFINITY : k;  // NaN ranks below every number
    }
    __syncthreads();
    float mx = -INFINITY, sum = 0.f;  // softmax statistics over all N logits (warp 0)
    if (warp == 0) {
      if (!SIGMOID) {
        for (int i = lane; i < N; i += 32) mx = fmaxf(mx, key[i]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        for (int i = lane; i < N; i += 32) sum += __expf(key[i] - mx);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      }
      uint32_t allowed = 0xffffffffu;  // node-limited routing: each node's largest key, then the allowed nodes
      if (a.nodes > 0) {
        float nmax[kMaxRouteNodes];
#pragma unroll
        for (int g = 0; g < kMaxRouteNodes; ++g) {
          float m = -INFINITY;
          if (g < a.nodes)
            for (int i = g * a.per_node + lane; i < (g + 1) * a.per_node; i += 32) m = fmaxf(m, key[i]);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          nmax[g] = m;
        }
        allowed = choose_nodes(nmax, a.nodes, a.max_nodes);
      }
      if (lane == 0) allowed_s = allowed;
    }
    __syncthreads();
    const uint32_t allowed = allowed_s;
    auto ok = [&](int i) { return a.nodes <= 0 || ((allowed >> (i / a.per_node)) & 1u); };
    if (tid < N && ok(tid)) {
      const float ki = key[tid];
      int rank = 0;
      if (a.nodes <= 0) {
#pragma unroll 8
        for (int j = 0; j < N; ++j) {
          const float kj = key[j];
          rank += (kj > ki || (kj == ki && j < tid)) ? 1 : 0;
        }
      } else {
        for (int j = 0; j < N; ++j) {
          const float kj = key[j];
          rank += (ok(j) && (kj > ki || (kj == ki && j < tid))) ? 1 : 0;
        }
      }
      if (rank < K) sel[rank] = tid;
    }
    __syncthreads();
    if (warp == 0 && lane == 0) {
      float ss[8], tot = 0.f;
      for (int k = 0; k < K; ++k) {
        const int i = sel[k];
        ss[k] = SIGMOID ? sval[i] : __expf(key[i] - mx) / sum;
        tot += ss[k];
      }
      for (int k = 0; k < K; ++k) {
        a.idx[static_cast<size_t>(t) * K + k] = sel[k];
        a.gate[static_cast<size_t>(t) * K + k] = SIGMOID ? ss[k] / tot : ss[k];
      }
      __threadfence();
      const uint32_t last = atomicAdd(a.done_counter, 1u) == static_cast<uint32_t>(T - 1) ? 1u : 0u;
      __threadfence();
      for (int q = 0; q < kRouteCluster; ++q) st_cluster_u32(mapa_shared(smem_u32(&is_last), q), last);
    }
  }
  cluster_sync();  // every CTA of the cluster knows whether its token was the last
  if (!is_last) return;
  // ---- the last cluster: tables and permutation of the whole batch ----
  __threadfence();
  for (int i = tid; i < N * 4; i += kRouteThreads) masks[i] = 0u;
  for (int i = tid; i < N; i += kRouteThreads) cnt[i] = 0;
  __syncthreads();
  if (tid < T) {
    for (int k = 0; k < K; ++k) {
      const int ex = __ldcg(a.idx + static_cast<size_t>(tid) * K + k);
      dst[tid * K + k] = ex;
      atomicOr(&masks[ex * 4 + (tid >> 5)], 1u << (tid & 31));
      atomicAdd(&cnt[ex], 1);
    }
  }
  __syncthreads();
  if (warp == 0) {  // lane l owns experts l * per .. l * per + per - 1
    const int per = (N + 31) >> 5;
    const int e0 = min(N, lane * per), e1 = min(N, e0 + per);
    int o = 0, mo = 0, m1 = 0;
    for (int ex = e0; ex < e1; ++ex) {
      o += cnt[ex];
      mo += (cnt[ex] + kExpertRowAlign - 1) / kExpertRowAlign;
      m1 += (cnt[ex] + 127) >> 7;
    }
#pragma unroll
    for (int sh = 1; sh < 32; sh <<= 1) {  // inclusive scans over the lanes
      const int po = __shfl_up_sync(0xffffffffu, o, sh), pm = __shfl_up_sync(0xffffffffu, mo, sh),
                p1 = __shfl_up_sync(0xffffffffu, m1, sh);
      if (lane >= sh) {
        o += po;
        mo += pm;
        m1 += p1;
      }
    }
    if (lane == 31) {
      roff[N] = o;
      mt[N] = mo;
      rstart[N] = mo * kExpertRowAlign;
      mt128[N] = m1;
    }
    for (int ex = e1 - 1; ex >= e0; --ex) {  // down from the inclusive sums
      o -= cnt[ex];
      mo -= (cnt[ex] + kExpertRowAlign - 1) / kExpertRowAlign;
      m1 -= (cnt[ex] + 127) >> 7;
      roff[ex] = o;
      mt[ex] = mo;
      rstart[ex] = mo * kExpertRowAlign;
      mt128[ex] = m1;
    }
  }
  __syncthreads();
  const bool lead = r == 0;
  if (lead) {
    if (tid < 2) p.tile_ctr[tid] = 0;
    if (tid == 0) *a.done_counter = 0u;  // every token has been counted
    for (int ex = tid; ex <= N; ex += kRouteThreads) {
      rt.offsets[ex] = roff[ex];
      rt.row_start[ex] = rstart[ex];
      rt.mtile_start[ex] = mt[ex];
      rt.mtile128_start[ex] = mt128[ex];
      if (ex < N) {
        rt.counts[ex] = cnt[ex];
        rt.block_counts[ex] = 0;
      }
    }
  }
  if (tid < T) {
    const int w = tid >> 5;
    const uint32_t below = (1u << (tid & 31)) - 1u;
    for (int k = 0; k < K; ++k) {
      const int ex = dst[tid * K + k];
      int rank = __popc(masks[ex * 4 + w] & below);
      for (int ww = 0; ww < w; ++ww) rank += __popc(masks[ex * 4 + ww]);
      const int prow = rstart[ex] + rank;
      dst[tid * K + k] = prow;  // this thread's own entries only
      if (lead) {
        p.src[roff[ex] + rank] = tid;
        p.slot_of[static_cast<size_t>(tid) * K + k] = prow;
        p.gate_perm[prow] = __ldcg(a.gate + static_cast<size_t>(tid) * K + k);
      }
    }
  }
  if (!p.gather) return;
  __syncthreads();
  // one warp per (token, slot) pair over the cluster's 64 warps, up to three
  // pairs at a time with all of their loads out before any store (a 32-token
  // batch with K = 6 gives each warp three 4 KB rows; one row per round trip
  // took 4.6 us, a warp per token row left half of the CTAs idle)
  const int nvec = d >> 3;
  constexpr int kW = kRouteCluster * (kRouteThreads / 32);
  for (int q0 = r * (kRouteThreads / 32) + warp; q0 < T * K; q0 += 3 * kW) {
    for (int c = lane; c < nvec; c += 32 * 4) {
      uint4 v[3][4];
#pragma unroll
      for (int pr = 0; pr < 3; ++pr) {
        const int q = q0 + pr * kW;
        const uint4* srow = reinterpret_cast<const uint4*>(x + static_cast<size_t>(q < T * K ? q / K : 0) * d);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          if (q < T * K && c + 32 * u < nvec) v[pr][u] = __ldg(srow + c + 32 * u);
      }
#pragma unroll
      for (int pr = 0; pr < 3; ++pr) {
        const int q = q0 + pr * kW;
        if (q < T * K) {
          uint4* drow = reinterpret_cast<uint4*>(p.x_perm + static_cast<size_t>(dst[q]) * d);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (c + 32 * u < nvec) drow[c + 32 * u] = v[pr][u];
        }
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
  // every operand in its own register (an array filled at a running index lived in local memory)
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
    for (int k = 0; k < 8; ++k)
      vy[k] = k < K ? __ldcg(reinterpret_cast<const uint4*>(a.y + static_cast<size_t>(slots[k]) * a.d + col)) : vx;
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
    *reinterpret_cast<uint4*>(a.out + static_cast<size_t>(t) * a.d + col) = o;
  }
}

}  // namespace fgs
