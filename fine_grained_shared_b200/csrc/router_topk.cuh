// router_topk.cuh -- step 1 and 2 of the layer: affinity logits on the
// tensor cores, softmax or sigmoid, top-K in registers, per-block expert
// histogram and (in the last CTA to finish) the expert-offset scan; the same
// steps on the CUDA cores for small batches; and the auxiliary-loss-free
// update of the selection biases from the per-expert counts.
//
// DeepSeekMoE (arXiv 2401.06066), Abstract: each token activates mK of the mN
// fine-grained routed experts.  DeepSeek-V3 technical report, section 2
// ("Auxiliary-Loss-Free Load Balancing"): per-expert biases steer which
// experts are chosen; every token keeps its K experts (no dropping).
//
// One CTA owns 128 tokens.  Warp 0 streams x[128 tokens, 64-column k-block]
// and e[mN (padded to 16), 64] into shared memory with TMA (128-byte
// swizzle); warp 1 issues tcgen05.mma (M = 128, N = mN padded) accumulating
// the logits z in TMEM; warps 2-5 (one TMEM lane = one token each) read the
// row of logits back and keep the K best keys in registers.
#pragma once

#include "sm100.cuh"

namespace fgs {

constexpr int kRouterThreads = 192;
// Pipeline depth: the ring holds kRouterMaxStages stages when they fit in
// about 200 KB of shared memory (mN <= 128), else 4.  6 stages x 2 copies stay
// within the 12 bulk copies in flight per CTA that every kernel here keeps
// to (measured on the 16B prefill layer: 0.064 ms against 0.065 with 4).
constexpr int kRouterMaxStages = 6;
__host__ __device__ constexpr int router_stages(int Npad) {
  return (16384 + Npad * 128) * kRouterMaxStages <= 200 * 1024 ? kRouterMaxStages : 4;
}
constexpr int kRouterBM = 128;
constexpr int kBK = 64;  // bf16 elements per 128-byte swizzle row
// Every expert's rows start on a multiple of this in the permuted row space,
// so that no 256-row GEMM tile (a CTA pair's tile) straddles two experts.
constexpr int kExpertRowAlign = 256;

struct RouterArgs {
  int T, N, Npad, num_kb, nblk;
  uint32_t tmem_cols;
  const float* logit_bias;   // [N] or null (softmax)
  const float* select_bias;  // [N] or null (sigmoid)
  int32_t* idx;              // [T, K]
  float* gate;               // [T, K]
  int32_t* block_counts;     // [nblk, N]; rewritten as per-block exclusive bases by the last CTA
  int32_t* counts;           // [N]
  int32_t* offsets;          // [N + 1] unpadded
  int32_t* row_start;        // [N + 1] start row of each expert, segments padded to kExpertRowAlign rows
  int32_t* mtile_start;      // [N + 1] prefix sum of ceil(count / kExpertRowAlign)
  int32_t* mtile128_start;   // [N + 1] prefix sum of ceil(count / 128)
  uint32_t* done_counter;    // CTAs finished; reset to 0 by the last CTA
  uint32_t* err;
  uint64_t timeout_ns;
  // node-limited routing (0 nodes: off): the mN experts sit on `nodes` nodes
  // in contiguous ranges of per_node; each token's K experts come from at
  // most max_nodes nodes, those holding its largest keys
  int nodes, per_node, max_nodes;
};

constexpr int kMaxRouteNodes = 16;

// The nodes a token may use: max_nodes rounds, each taking the unchosen node
// with the largest key maximum (ties to the lower node), as a bit mask.
__device__ __forceinline__ uint32_t choose_nodes(const float (&nmax)[kMaxRouteNodes], int nodes, int max_nodes) {
  uint32_t chosen = 0u;
  for (int m = 0; m < max_nodes; ++m) {
    float bv = -INFINITY;
    int bg = kMaxRouteNodes;
#pragma unroll
    for (int g = 0; g < kMaxRouteNodes; ++g) {
      if (g < nodes && !((chosen >> g) & 1u) && (nmax[g] > bv || (nmax[g] == bv && g < bg))) {
        bv = nmax[g];
        bg = g;
      }
    }
    chosen |= 1u << bg;
  }
  return chosen;
}

__host__ __device__ constexpr size_t router_smem_bytes(int Npad) {
  return 1024 + static_cast<size_t>(router_stages(Npad)) * (16384 + static_cast<size_t>(Npad) * 128) +
         8 * (2 * kRouterMaxStages + 2) + 16 + 4 * (256 + 256 + 256) + 64;
}

__device__ __forceinline__ void record_error(uint32_t* err, volatile int* abort, uint32_t site) {
  *abort = 1;
  atomicOr(err, kErrTimeout | (1u << (kErrSiteShift + site)));
}

// NL: node-limited routing -- a first pass over the token's logits in TMEM
// takes each node's largest key and picks the allowed nodes (choose_nodes);
// the top-K pass then skips the experts of the other nodes.  The softmax
// statistics still cover every expert.
template <int K, bool SIGMOID, bool NL>
__global__ void __launch_bounds__(kRouterThreads, 1)
    router_topk_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_e,
                       RouterArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int Bbytes = a.Npad * 128;
  uint8_t* sA = smem;
  const int S = router_stages(a.Npad);
  uint8_t* sB = smem + S * 16384;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + S * Bbytes);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;
  uint64_t* teardown = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(teardown + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* is_last = reinterpret_cast<int*>(tmem_slot + 2);
  int* hist = reinterpret_cast<int*>(tmem_slot + 4);
  float* bias = reinterpret_cast<float*>(hist + 256);
  int* scan_tmp = reinterpret_cast<int*>(bias + 256);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * kRouterBM;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(teardown, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, a.tmem_cols);
    tmem_relinquish();
  }
  pdl_wait();  // x, the biases and every output buffer belong to earlier kernels until here
  pdl_launch_dependents();
  for (int i = tid; i < 256; i += kRouterThreads) {
    hist[i] = 0;
    float b = 0.f;
    if (i < a.N) {
      if (SIGMOID) {
        if (a.select_bias) b = a.select_bias[i];
      } else {
        if (a.logit_bias) b = a.logit_bias[i];
      }
    }
    bias[i] = b;
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer ----------------
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_e);
    int s = 0, issued = 0;
    uint32_t ph = 0;
    for (int kb = 0; kb < a.num_kb; ++kb) {
      if (!mbar_wait(&empty[s], ph ^ 1u, a.timeout_ns, abort_flag)) {
        record_error(a.err, abort_flag, 0);
        break;
      }
      mbar_arrive_expect_tx(&full[s], 16384u + static_cast<uint32_t>(Bbytes));
      tma_load_2d(sA + s * 16384, &tm_x, &full[s], kb * kBK, m0);
      tma_load_2d(sB + s * Bbytes, &tm_e, &full[s], kb * kBK, 0);
      ++issued;
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
    }
    // make sure no copy is still landing in shared memory when the CTA exits
    for (int st = 0; st < S; ++st) {
      if (issued > st) {
        const int n = (issued - 1 - st) / S + 1;
        mbar_wait_drain(&full[st], static_cast<uint32_t>((n - 1) & 1), a.timeout_ns);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    const uint32_t idesc = idesc_bf16_f32(128, a.Npad);
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int kb = 0; kb < a.num_kb; ++kb) {
      if (!mbar_wait(&full[s], ph, a.timeout_ns, abort_flag)) {
        record_error(a.err, abort_flag, 1);
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + s * 16384));
      const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + s * Bbytes));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_bf16_ss(tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
      umma_commit(&empty[s]);
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
    }
    if (ok) umma_commit(acc_full);
    umma_commit(teardown);
    mbar_wait_drain(teardown, 0, a.timeout_ns);
  } else if (warp >= 2) {
    // ---------------- epilogue: one token per thread ----------------
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int t = m0 + r;
    bool ok = mbar_wait(acc_full, 0, a.timeout_ns, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) {
      if (lane == 0) record_error(a.err, abort_flag, 2);
    } else {
      tc_fence_after_sync();
      float tk[K], ts[K];
      int ti[K];
#pragma unroll
      for (int k = 0; k < K; ++k) {
        tk[k] = -INFINITY;
        ts[k] = 0.f;
        ti[k] = 0x7fffffff;
      }
      float mx = -INFINITY, sum = 0.f;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16);
      uint32_t allowed = 0xffffffffu;  // bit g: node g may hold a selected expert
      if (NL) {
        float nmax[kMaxRouteNodes];
#pragma unroll
        for (int g = 0; g < kMaxRouteNodes; ++g) nmax[g] = -INFINITY;
        for (int c0 = 0; c0 < a.Npad; c0 += 16) {
          uint32_t rr[16];
          tmem_ld16(tbase + c0, rr);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int col = c0 + j;
            if (col < a.N) {
              // the key exactly as the top-K pass below computes it
              const float z = __uint_as_float(rr[j]);
              float key = SIGMOID ? 1.f / (1.f + __expf(-z)) + bias[col] : z + bias[col];
              if (isnan(key)) key = -INFINITY;
              const int node = col / a.per_node;
#pragma unroll
              for (int g = 0; g < kMaxRouteNodes; ++g)
                if (g == node) nmax[g] = fmaxf(nmax[g], key);
            }
          }
        }
        allowed = choose_nodes(nmax, a.nodes, a.max_nodes);
      }
      for (int c0 = 0; c0 < a.Npad; c0 += 16) {
        uint32_t rr[16];
        tmem_ld16(tbase + c0, rr);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int col = c0 + j;
          if (col < a.N) {
            float z = __uint_as_float(rr[j]);
            float key, sv;
            if (SIGMOID) {
              sv = 1.f / (1.f + __expf(-z));
              key = sv + bias[col];
            } else {
              z += bias[col];
              if (z > mx) {
                sum = sum * __expf(mx - z) + 1.f;
                mx = z;
              } else {
                sum += __expf(z - mx);
              }
              key = z;  // softmax is monotone in z: rank on the logits
              sv = 0.f;
            }
            // a NaN key (a non-finite token or router row) ranks below every
            // number; the index order then still fills the K slots with
            // distinct experts in [0, N)
            if (isnan(key)) key = -INFINITY;
            if (NL && !((allowed >> (col / a.per_node)) & 1u)) continue;  // a node not chosen
            // insert (key, col) into the list ordered by (key descending,
            // index ascending); an element pushed down keeps competing by the
            // same order, so ties always go to the lower expert index
            float v = key, vs = sv;
            int vi = col;
#pragma unroll
            for (int k = 0; k < K; ++k) {
              const bool sw = (v > tk[k]) || (v == tk[k] && vi < ti[k]);
              const float t0 = tk[k], t1 = ts[k];
              const int t2 = ti[k];
              tk[k] = sw ? v : t0;
              ts[k] = sw ? vs : t1;
              ti[k] = sw ? vi : t2;
              v = sw ? t0 : v;
              vs = sw ? t1 : vs;
              vi = sw ? t2 : vi;
            }
          }
        }
      }
      if (t < a.T) {
        float g[K];
        if (SIGMOID) {
          float tot = 0.f;
#pragma unroll
          for (int k = 0; k < K; ++k) tot += ts[k];
#pragma unroll
          for (int k = 0; k < K; ++k) g[k] = ts[k] / tot;
        } else {
          const float inv = 1.f / sum;
#pragma unroll
          for (int k = 0; k < K; ++k) g[k] = __expf(tk[k] - mx) * inv;
        }
#pragma unroll
        for (int k = 0; k < K; ++k) {
          a.idx[static_cast<size_t>(t) * K + k] = ti[k];
          a.gate[static_cast<size_t>(t) * K + k] = g[k];
          if (ti[k] < a.N) atomicAdd(&hist[ti[k]], 1);
        }
      }
    }
    tc_fence_before_sync();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, a.tmem_cols);
  }

  // ---------------- per-block histogram and the last-CTA scan ----------------
  for (int e = tid; e < a.N; e += kRouterThreads)
    a.block_counts[static_cast<size_t>(blockIdx.x) * a.N + e] = hist[e];
  __threadfence();
  __syncthreads();
  if (tid == 0) *is_last = (atomicAdd(a.done_counter, 1u) == static_cast<uint32_t>(a.nblk - 1));
  __syncthreads();
  if (!*is_last) return;
  __threadfence();
  for (int e = tid; e < a.N; e += kRouterThreads) {
    // exclusive scan of expert e's column over the blocks, 16 independent
    // loads in flight at a time (the column is strided by N in memory)
    int run = 0;
    for (int b0 = 0; b0 < a.nblk; b0 += 16) {
      int v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        v[i] = (b0 + i < a.nblk) ? __ldcg(a.block_counts + static_cast<size_t>(b0 + i) * a.N + e) : 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (b0 + i < a.nblk) a.block_counts[static_cast<size_t>(b0 + i) * a.N + e] = run;
        run += v[i];
      }
    }
    a.counts[e] = run;
    scan_tmp[e] = run;
  }
  __syncthreads();
  if (tid == 0) {
    int o = 0, ro = 0, mo = 0, m128 = 0;
    for (int e = 0; e < a.N; ++e) {
      a.offsets[e] = o;
      a.row_start[e] = ro;
      a.mtile_start[e] = mo;
      a.mtile128_start[e] = m128;
      const int c = scan_tmp[e];
      const int mt = (c + kExpertRowAlign - 1) / kExpertRowAlign;
      o += c;
      mo += mt;
      m128 += (c + 127) / 128;
      ro += mt * kExpertRowAlign;
    }
    a.offsets[a.N] = o;
    a.row_start[a.N] = ro;
    a.mtile_start[a.N] = mo;
    a.mtile128_start[a.N] = m128;
    *a.done_counter = 0u;
  }
}

}  // namespace fgs

namespace fgs {

// ---------------------------------------------------------------------------
// Small batches (T <= kSmallRouterMaxT) on the CUDA cores.  The tensor-core
// router gives a 128-token block to one CTA, so a decode batch of a few dozen
// tokens would run on a single SM walking d serially.  Here the grid is
// (token, group of kSmallRouterGroup experts): each warp computes one
// expert's logit as a dot product, every lane issuing its loads for a whole
// 2048-column pass at once (instead of one CTA pulling all mN experts' rows
// through its lanes: 16B decode, T = 32, 25 -> 17 us), and writes it to a
// per-token row of logits.  The last of a token's CTAs to finish (a
// per-token counter) picks that token's top K by K rounds of a warp argmax
// ordered by (key descending, index ascending); the last token to be
// finished counts the selected experts of every 128-token block from the
// written indices (shared-memory integer atomics: exact) and runs the same
// scan as the tensor-core router.  Both counters are reset by their last
// arriver, so no buffer needs clearing between calls.
// ---------------------------------------------------------------------------
// A 16-byte read-only global load that the compiler keeps in program order
// with the other such loads, so a batch of them is in flight together.
__device__ __forceinline__ uint4 ldg_v4_ordered(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

constexpr int kSmallRouterMaxT = 256;
constexpr int kSmallRouterThreads = 256;
constexpr int kSmallRouterGroup = 8;   // experts per CTA: one per warp
static_assert(kSmallRouterThreads / 32 == kSmallRouterGroup, "one warp per expert of the group");
constexpr int kSmallRouterPass = 8;    // 16-byte vectors per lane per pass (2048 columns)

// Token t's selection by one warp from its N logits zrow (step 2 of the layer):
// the keys (softmax: logit + logit bias; sigmoid: s + selection bias, NaN
// ranked below every number), the softmax statistics over all N, the allowed
// nodes under node-limited routing, then K rounds of a warp argmax ordered by
// (key descending, index ascending); writes idx[t, :] and gate[t, :].  key and
// sval are shared-memory rows of at least N floats; ZGLOBAL: zrow is in global
// memory, written by other CTAs (read through L2).  lbias / sbias: the logit
// and selection biases (either may be null).
template <bool SIGMOID, bool ZGLOBAL>
__device__ __forceinline__ void select_token_warp(int t, int K, const RouterArgs& a, const float* zrow, float* key,
                                                  float* sval, const float* lbias, const float* sbias) {
  const int lane = threadIdx.x & 31;
  for (int i = lane; i < a.N; i += 32) {
    const float z = ZGLOBAL ? __ldcg(zrow + i) : zrow[i];
    if (SIGMOID) {
      const float sv = 1.f / (1.f + __expf(-z));
      sval[i] = sv;
      const float k = sv + (sbias ? sbias[i] : 0.f);
      key[i] = isnan(k) ? -INFINITY : k;  // NaN ranks below every number
    } else {
      const float k = z + (lbias ? lbias[i] : 0.f);  // softmax is monotone in z
      key[i] = isnan(k) ? -INFINITY : k;
    }
  }
  __syncwarp();
  // softmax statistics over all N logits (softmax mode)
  float mx = -INFINITY, sum = 0.f;
  if (!SIGMOID) {
    for (int i = lane; i < a.N; i += 32) mx = fmaxf(mx, key[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    for (int i = lane; i < a.N; i += 32) sum += __expf(key[i] - mx);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  }
  // node-limited routing: each node's largest key, then the allowed nodes
  uint32_t allowed = 0xffffffffu;
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
  uint32_t taken = 0;  // bit j: this lane's expert lane + 32 * j is already selected
  int sel[8];
  float sel_s[8];
  float tot = 0.f;
  for (int k = 0; k < K; ++k) {
    float bk = -INFINITY;
    int bi = 0x7fffffff;
    for (int j = 0, i = lane; i < a.N; ++j, i += 32) {
      if (taken & (1u << j)) continue;
      if (a.nodes > 0 && !((allowed >> (i / a.per_node)) & 1u)) continue;
      const float v = key[i];
      if (v > bk || (v == bk && i < bi)) {
        bk = v;
        bi = i;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bk || (ov == bk && oi < bi)) {
        bk = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    sel[k] = bi;
    sel_s[k] = SIGMOID ? sval[bi] : __expf(bk - mx) / sum;
    tot += sel_s[k];
  }
  if (lane == 0) {
    for (int k = 0; k < K; ++k) {
      a.idx[static_cast<size_t>(t) * K + k] = sel[k];
      a.gate[static_cast<size_t>(t) * K + k] = SIGMOID ? sel_s[k] / tot : sel_s[k];
    }
  }
}

struct SmallRouterArgs {
  float* logits;          // [T, N] fp32 scratch
  uint32_t* token_done;   // [T] CTAs finished per token, zero between calls
};

template <bool SIGMOID>
__global__ void __launch_bounds__(kSmallRouterThreads)
    router_small_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ e, int d, int K,
                        RouterArgs a, SmallRouterArgs sa) {
  static_assert(kSmallRouterMaxT <= 2 * 128, "the last CTA's histogram holds two 128-token blocks");
  __shared__ float key[256], sval[256];
  __shared__ int is_last;
  __shared__ int scan_tmp[256];
  __shared__ int hist[2][256];
  const int t = blockIdx.x, grp = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();
  pdl_launch_dependents();
  // ---- the logit of this warp's expert ----
  {
    const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d);
    const int nvec = d >> 3;
    const int i = grp * kSmallRouterGroup + warp;
    if (i < a.N) {
      const uint4* er = reinterpret_cast<const uint4*>(e + static_cast<size_t>(i) * d);
      float acc = 0.f;
      for (int c0 = 0; c0 < nvec; c0 += 32 * kSmallRouterPass) {
        uint4 xv[kSmallRouterPass], ev[kSmallRouterPass];
        // all 2 x kSmallRouterPass loads issue before any arithmetic; a column
        // past the row reads column 0 of the same rows and is zeroed in x
#pragma unroll
        for (int j = 0; j < kSmallRouterPass; ++j) {
          const int c = c0 + lane + 32 * j;
          const int cc = c < nvec ? c : 0;
          xv[j] = ldg_v4_ordered(xr + cc);
          ev[j] = ldg_v4_ordered(er + cc);
        }
#pragma unroll
        for (int j = 0; j < kSmallRouterPass; ++j) {
          if (c0 + lane + 32 * j >= nvec) xv[j] = make_uint4(0, 0, 0, 0);
          const uint32_t xw[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w};
          const uint32_t w[4] = {ev[j].x, ev[j].y, ev[j].z, ev[j].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc = fmaf(bf16lo(xw[q]), bf16lo(w[q]), acc);
            acc = fmaf(bf16hi(xw[q]), bf16hi(w[q]), acc);
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) sa.logits[static_cast<size_t>(t) * a.N + i] = acc;
    }
  }
  // ---- the last of the token's CTAs picks its top K ----
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = (atomicAdd(sa.token_done + t, 1u) == gridDim.y - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  if (tid == 0) sa.token_done[t] = 0u;  // every CTA of this token has counted itself
  if (warp == 0)
    select_token_warp<SIGMOID, true>(t, K, a, sa.logits + static_cast<size_t>(t) * a.N, key, sval, a.logit_bias,
                                     a.select_bias);
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = (atomicAdd(a.done_counter, 1u) == static_cast<uint32_t>(gridDim.x - 1));
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // every token's selection is written: count them per 128-token block
  for (int i = tid; i < 2 * 256; i += kSmallRouterThreads) (&hist[0][0])[i] = 0;
  __syncthreads();
  const int TK = a.T * K;
  for (int i = tid; i < TK; i += kSmallRouterThreads) atomicAdd(&hist[(i / K) >> 7][__ldcg(a.idx + i)], 1);
  __syncthreads();
  for (int ex = tid; ex < a.N; ex += kSmallRouterThreads) {
    int run = 0;
    for (int b = 0; b < a.nblk; ++b) {
      a.block_counts[static_cast<size_t>(b) * a.N + ex] = run;  // exclusive base of block b
      run += hist[b][ex];
    }
    a.counts[ex] = run;
    scan_tmp[ex] = run;
  }
  __syncthreads();
  if (tid == 0) {
    int o = 0, ro = 0, mo = 0, m128 = 0;
    for (int ex = 0; ex < a.N; ++ex) {
      a.offsets[ex] = o;
      a.row_start[ex] = ro;
      a.mtile_start[ex] = mo;
      a.mtile128_start[ex] = m128;
      const int c = scan_tmp[ex];
      const int mt = (c + kExpertRowAlign - 1) / kExpertRowAlign;
      o += c;
      mo += mt;
      m128 += (c + 127) / 128;
      ro += mt * kExpertRowAlign;
    }
    a.offsets[a.N] = o;
    a.row_start[a.N] = ro;
    a.mtile_start[a.N] = mo;
    a.mtile128_start[a.N] = m128;
    *a.done_counter = 0u;
  }
}

// ---------------------------------------------------------------------------
// Auxiliary-loss-free load balancing (DeepSeek-V3 technical report summary,
// section 2): after a step, every expert's selection bias moves by gamma
// according to whether the expert was overloaded or underloaded.  With the
// step's per-expert loads (the router's counts): b_i += gamma * sign(mean -
// load_i), the comparison made on integers (load_i * N against the total).
// One thread per expert; the total comes from a block reduction.
// ---------------------------------------------------------------------------
constexpr int kBiasThreads = 256;

static __global__ void __launch_bounds__(kBiasThreads)
    bias_update_kernel(float* __restrict__ bias, const int32_t* __restrict__ counts, int N, float gamma) {
  __shared__ long long part[kBiasThreads / 32];
  const int tid = threadIdx.x;
  long long sum = 0;
  for (int i = tid; i < N; i += kBiasThreads) sum += counts[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if ((tid & 31) == 0) part[tid >> 5] = sum;
  __syncthreads();
  long long total = 0;
#pragma unroll
  for (int w = 0; w < kBiasThreads / 32; ++w) total += part[w];
  for (int i = tid; i < N; i += kBiasThreads) {
    const long long scaled = static_cast<long long>(counts[i]) * N;  // load_i * N vs total = mean * N
    const float step = scaled < total ? gamma : scaled > total ? -gamma : 0.f;
    bias[i] = bias[i] + step;
  }
}

}  // namespace fgs
