// decode_ffn.cuh -- steps 4-5 of the layer (the gate/up GEMM + SwiGLU and the
// down GEMM + gate scale, shared and routed experts) for a decode batch, in
// one persistent launch.
//
// A decode batch (T <= 64 tokens) makes the expert GEMMs a stream of weights:
// every touched expert's W_gate, W_up and W_down cross HBM once, and at 32
// token rows per tile the MMAs are idle most of the time.  The work is the
// whole tiles [128 weight rows x <= 32 token rows] of four kinds, numbered in
// this order:
//   0  shared gate/up   (weight block wb of the K_s I_s columns, token block tb)
//   1  routed gate/up   (expert g, weight block wb of I, token block tb)
//   2  shared down      (weight block wb of d, token block tb)
//   3  routed down      (expert g, weight block wb of d, token block tb)
// and each of the persistent CTAs (one per SM) takes the next tile from a
// global counter until none is left.  Whole tiles keep every result
// deterministic (no tile's sum is split between CTAs); taking them in turn
// evens out the CTAs' bytes to within one tile, and a CTA that finishes its
// gate/up tiles streams down-projection weights while other CTAs still finish
// theirs (the two GEMMs as separate launches left every SM idle from its own
// last gate/up tile to the last one of the grid, and then for the start of
// the down launch).  A down tile reads the rows of H of its token block, so
// before it loads them the producer waits for that block's readiness counter,
// which every epilogue warp raises once per finished gate/up tile (4 n_wb per
// block when complete).  The numbering puts all gate/up tiles first, so the
// tile a CTA waits on is always held by a running CTA: no wait can be circular.
// The shared gate/up tiles need neither the router nor the permutation, so
// they also run ahead of the grid dependency wait.
//
// One CTA per SM, 192 threads:
//   warp 0   scheduler and TMA producer: takes tiles, publishes each in a
//            shared-memory ring of work items, and streams its k-blocks into
//            a ring of 4 stages of 40 KB (a gate/up stage: the W_gate and W_up
//            boxes [128 rows, 64] and the token box [32 rows, 64]; a down
//            stage: two k-blocks of the W_down box and the H box), 128-byte
//            swizzle.  Weights are read once, so their loads carry an L2
//            evict-first policy.
//   warp 1   allocates all 512 TMEM columns (eight accumulator buffers of 64:
//            gate and up, or down alone); one lane issues the MMAs
//   warps 2-5 epilogue: thread r holds weight row r of the accumulator, i.e.
//            one output column for the tile's (up to) 32 tokens
// The last CTA to finish resets the tile counter and the readiness counters
// for the next launch.
#pragma once

#include "sm100.cuh"

namespace fgs {

constexpr int kFfnThreads = 192;
constexpr int kFfnTB = 32;   // token rows per tile (MMA N)
constexpr int kFfnWB = 128;  // weight rows per tile (MMA M)
constexpr int kFfnBK = 64;   // k-block: one 128-byte swizzle row of bf16
constexpr uint32_t kFfnBoxW = kFfnWB * kFfnBK * 2;  // 16 KB
constexpr uint32_t kFfnBoxX = kFfnTB * kFfnBK * 2;  // 4 KB
constexpr int kFfnStages = 4;
constexpr uint32_t kFfnStage = 2 * (kFfnBoxW + kFfnBoxX);  // 40 KB: two down k-blocks, or one gate/up k-block
static_assert(2 * kFfnBoxW + kFfnBoxX <= kFfnStage, "a gate/up k-block fits a stage");
constexpr int kFfnAccBufs = 8;                         // accumulator buffers of 64 columns
constexpr uint32_t kFfnTmemCols = 64 * kFfnAccBufs;    // all 512 columns: one CTA per SM
constexpr int kFfnItems = 8;                           // work-item ring
constexpr int kFfnMaxBlocks = 512;                     // token blocks with a readiness counter
constexpr int kFfnMaxExperts = 256;
// TMA box heights the host must encode
constexpr uint32_t kFfnBoxRowsW = kFfnWB;
constexpr uint32_t kFfnBoxRowsX = kFfnTB;

// the work counters: [0] next tile, [1] CTAs finished, [2 ...] readiness per token block
constexpr size_t ffn_counter_bytes() { return static_cast<size_t>(2 + kFfnMaxBlocks) * 4; }

struct FfnItem {
  int kind;    // 0-3 as above; -1: no tile left
  int g, wb;   // expert (routed), weight block
  int row0;    // first token row (of x / X_perm / Hs / H)
  int nvalid;  // token rows of the block that exist
  int nkb;     // k-blocks of the tile
  int ready;   // the readiness counter it raises (gate/up) or waits on (down)
};

__host__ __device__ constexpr size_t ffn_smem_bytes() {
  return 1024 + static_cast<size_t>(kFfnStages) * kFfnStage +
         8 * (2 * kFfnStages + 2 * kFfnAccBufs + 2 * kFfnItems + 2) + 16 + sizeof(FfnItem) * kFfnItems +
         4 * (3 * (kFfnMaxExperts + 8));
}
static_assert(ffn_smem_bytes() <= 232448, "shared memory");
// all 512 TMEM columns per CTA: shared memory keeps two of these CTAs off one
// SM (one would wait in tcgen05.alloc until the other ends)
static_assert(2 * ffn_smem_bytes() > 233472, "two CTAs would fit on one SM");

struct FfnArgs {
  int T;                       // tokens
  int G;                       // routed experts (0: no routed tiles)
  int sh_blocks;               // shared token blocks (0: no shared tiles)
  int n_wb_gu, n_wb_dn;        // routed weight blocks: over I (gate/up), over d (down)
  int kb_gu, kb_dn;            // routed k-blocks: over d (gate/up), over I (down)
  int sh_n_wb_gu, sh_n_wb_dn;  // shared weight blocks: over K_s I_s, over d
  int sh_J, sh_kb_per_j, sh_k_per_j;  // shared down k loop: K_s experts x I_s / 64 k-blocks, I_s columns each
  const int32_t* counts;       // [G] rows of each expert
  const int32_t* row_start;    // [G + 1] first row of each expert in X_perm / H / Y
  const float* row_scale;      // [rows] the gate g of each row of Y
  __nv_bfloat16* h;            // [rows, I]
  __nv_bfloat16* hs;           // [T, K_s I_s]
  __nv_bfloat16* y;            // [rows, d]
  __nv_bfloat16* ys;           // [T, d]
  int I, sh_cols, d;           // columns of H, Hs, Y / Ys
  uint32_t* ctr;               // ffn_counter_bytes(), zero between launches
  uint32_t* err;
  uint64_t timeout_ns;
  int debug_wait;              // test only: CTA 0's MMA lane waits 20 ms on a barrier nothing arrives on
};

__device__ __forceinline__ void ffn_record_error(uint32_t* err, volatile int* abort, uint32_t site) {
  *abort = 1;
  atomicOr(err, kErrTimeout | (1u << (kErrSiteShift + site)));
}

// Waits (bounded) until the readiness counter reaches target; gives up early once any CTA of the launch
// has recorded an error (the tiles it waits for may belong to a CTA that stopped).
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p);
__device__ __forceinline__ bool ffn_wait_ready(const uint32_t* ctr, uint32_t target, const uint32_t* err,
                                               volatile int* abort, uint64_t timeout_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (ld_acquire_u32(ctr) < target) {
    if (*abort || *reinterpret_cast<const volatile uint32_t*>(err) != 0u || globaltimer_ns() - t0 > timeout_ns)
      return false;
    __nanosleep(64);
  }
  return true;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Generic-proxy writes of this thread (the rows of H), ordered before later
// async-proxy (TMA) reads of global memory.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// 32 lanes x 32 columns of 32-bit TMEM cells
__device__ __forceinline__ void ffn_tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[16];
  tmem_ld16(taddr, r);
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
  tmem_ld16(taddr + 16, r);
#pragma unroll
  for (int j = 0; j < 16; ++j) v[16 + j] = __uint_as_float(r[j]);
}

// Gate/up maps: tmWg / tmWu the routed experts' W_gate / W_up as [G][I][d],
// tmX X_perm, tmWsg / tmWsu the shared experts' as [1][K_s I_s][d], tmXs x.
// Down maps: tmWd W_down as [G][d][I], tmH H, tmWsd W_down,s as
// [K_s][d][I_s], tmHs Hs.  Weight boxes 128 rows, token boxes 32 rows, all 64
// columns wide.  Maps of an absent part are never read.
__global__ void __launch_bounds__(kFfnThreads, 1)
    decode_ffn_kernel(const __grid_constant__ CUtensorMap tmWg, const __grid_constant__ CUtensorMap tmWu,
                      const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWsg,
                      const __grid_constant__ CUtensorMap tmWsu, const __grid_constant__ CUtensorMap tmXs,
                      const __grid_constant__ CUtensorMap tmWd, const __grid_constant__ CUtensorMap tmH,
                      const __grid_constant__ CUtensorMap tmWsd, const __grid_constant__ CUtensorMap tmHs,
                      FfnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kFfnStages * kFfnStage);
  uint64_t* empty = full + kFfnStages;
  uint64_t* acc_full = empty + kFfnStages;       // [kFfnAccBufs]
  uint64_t* acc_empty = acc_full + kFfnAccBufs;  // [kFfnAccBufs]
  uint64_t* item_full = acc_empty + kFfnAccBufs;  // [kFfnItems]
  uint64_t* item_empty = item_full + kFfnItems;   // [kFfnItems]
  uint64_t* teardown = item_empty + kFfnItems;
  uint64_t* never = teardown + 1;  // test only: a barrier nothing arrives on
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  FfnItem* items = reinterpret_cast<FfnItem*>(tmem_slot + 4);
  int32_t* s_tbs = reinterpret_cast<int32_t*>(items + kFfnItems);  // [G + 1] prefix of 32-token blocks
  int32_t* s_rows = s_tbs + kFfnMaxExperts + 8;                       // [G]
  int32_t* s_cnt = s_rows + kFfnMaxExperts + 8;                       // [G]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kFfnStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < kFfnAccBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);  // one arrive per epilogue warp
    }
    for (int i = 0; i < kFfnItems; ++i) {
      mbar_init(&item_full[i], 1);
      mbar_init(&item_empty[i], 5);  // the MMA lane and the four epilogue warps
    }
    mbar_init(teardown, 1);
    mbar_init(never, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kFfnTmemCols);
    tmem_relinquish();
  }
  pdl_launch_dependents();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  uint32_t* const next_tile = a.ctr;
  uint32_t* const ctas_done = a.ctr + 1;
  uint32_t* const ready = a.ctr + 2;

  if (warp == 0) {
    // ------------------------ scheduler and TMA producer ------------------------
    const uint64_t pol_w = l2_policy_evict_first();
    const int sb = a.sh_blocks;
    const long long n_gsh = static_cast<long long>(a.sh_n_wb_gu) * sb;
    long long n_gr = 0, n_dsh = static_cast<long long>(a.sh_n_wb_dn) * sb, n_dr = 0;
    bool have_tables = false;
    int s = 0, issued = 0, it = 0;
    uint32_t ph = 0, it_ph = 0;
    bool stop = false;
    if (lane == 0) {
      if (sb) {
        tma_prefetch_desc(&tmWsg);
        tma_prefetch_desc(&tmWsu);
        tma_prefetch_desc(&tmXs);
      }
    }
    // routed tile t of a space with n_wb weight blocks per expert: weight-block major within an expert
    auto routed = [&](long long t, int n_wb, FfnItem& f) {
      int lo = 0, hi = a.G;  // largest g with s_tbs[g] * n_wb <= t
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (static_cast<long long>(s_tbs[mid]) * n_wb <= t) lo = mid;
        else hi = mid;
      }
      const int ntb = s_tbs[lo + 1] - s_tbs[lo];
      const int local = static_cast<int>(t - static_cast<long long>(s_tbs[lo]) * n_wb);
      f.g = lo;
      f.wb = local / ntb;
      const int tb = local - f.wb * ntb;
      f.row0 = s_rows[lo] + tb * kFfnTB;
      f.nvalid = min(kFfnTB, s_cnt[lo] - tb * kFfnTB);
      f.ready = sb + s_tbs[lo] + tb;
    };
    auto shared_tile = [&](long long t, FfnItem& f) {
      f.g = 0;
      f.wb = static_cast<int>(t / sb);
      const int tb = static_cast<int>(t - static_cast<long long>(f.wb) * sb);
      f.row0 = tb * kFfnTB;
      f.nvalid = min(kFfnTB, a.T - tb * kFfnTB);
      f.ready = tb;
    };
    while (!stop) {
      long long w = 0;
      if (lane == 0) w = static_cast<long long>(atomicAdd(next_tile, 1u));
      w = __shfl_sync(0xffffffffu, w, 0);
      if (w >= n_gsh && !have_tables) {
        // the router's tables and the permuted rows are complete from here
        pdl_wait();
        // 32-token blocks of each expert, prefix-summed (a warp scan of per-lane sums)
        int run = 0, loc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int g = lane * 8 + i;
          const int cnt = g < a.G ? a.counts[g] : 0;
          loc[i] = (cnt + kFfnTB - 1) / kFfnTB;
          if (g < a.G) {
            s_cnt[g] = cnt;
            s_rows[g] = a.row_start[g];
          }
          run += loc[i];
        }
        int incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        int ex = incl - run;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int g = lane * 8 + i;
          if (g <= a.G) s_tbs[g] = ex;
          ex += loc[i];
        }
        if (lane == 31 && a.G == kFfnMaxExperts) s_tbs[kFfnMaxExperts] = incl;
        __syncwarp();
        const long long tbs = a.G ? s_tbs[a.G] : 0;
        n_gr = tbs * a.n_wb_gu;
        n_dr = tbs * a.n_wb_dn;
        have_tables = true;
        if (lane == 0 && a.G) {
          tma_prefetch_desc(&tmWg);
          tma_prefetch_desc(&tmWu);
          tma_prefetch_desc(&tmX);
          tma_prefetch_desc(&tmWd);
          tma_prefetch_desc(&tmH);
        }
        if (lane == 0 && sb) {
          tma_prefetch_desc(&tmWsd);
          tma_prefetch_desc(&tmHs);
        }
      }
      FfnItem f{};
      f.kind = -1;
      {
        long long r = w;
        if (r < n_gsh) {
          f.kind = 0;
          shared_tile(r, f);
          f.nkb = a.kb_gu;
        } else if ((r -= n_gsh) < n_gr) {
          f.kind = 1;
          routed(r, a.n_wb_gu, f);
          f.nkb = a.kb_gu;
        } else if ((r -= n_gr) < n_dsh) {
          f.kind = 2;
          shared_tile(r, f);
          f.nkb = a.sh_J * a.sh_kb_per_j;
        } else if ((r -= n_dsh) < n_dr) {
          f.kind = 3;
          routed(r, a.n_wb_dn, f);
          f.nkb = a.kb_dn;
        }
      }
      if (lane == 0) {
        // publish the tile to the MMA lane and the epilogue
        if (!mbar_wait(&item_empty[it], it_ph ^ 1u, a.timeout_ns, abort_flag)) {
          ffn_record_error(a.err, abort_flag, 1);
          stop = true;
        } else {
          items[it] = f;
          mbar_arrive(&item_full[it]);
          if (++it == kFfnItems) {
            it = 0;
            it_ph ^= 1u;
          }
        }
        if (f.kind < 0) stop = true;
        if (!stop && f.kind >= 2) {
          // the down tile's rows of H: wait for every gate/up tile of its token block
          const uint32_t target = 4u * static_cast<uint32_t>(f.kind == 2 ? a.sh_n_wb_gu : a.n_wb_gu);
          if (!ffn_wait_ready(ready + f.ready, target, a.err, abort_flag, a.timeout_ns)) {
            ffn_record_error(a.err, abort_flag, 2);
            stop = true;
          }
          fence_proxy_async_global();
        }
        // stream the tile's k-blocks: one per gate/up stage, two per down stage
        const int per = f.kind >= 2 ? 2 : 1;
        for (int kb = 0; !stop && kb < f.nkb; kb += per) {
          if (!mbar_wait(&empty[s], ph ^ 1u, a.timeout_ns, abort_flag)) {
            ffn_record_error(a.err, abort_flag, 3);
            stop = true;
            break;
          }
          uint8_t* st = smem + s * kFfnStage;
          const int wrow = f.wb * kFfnWB;
          if (f.kind < 2) {
            const int kc = kb * kFfnBK;
            mbar_arrive_expect_tx(&full[s], 2 * kFfnBoxW + kFfnBoxX);
            tma_load_3d_hint(st, f.kind == 0 ? &tmWsg : &tmWg, &full[s], kc, wrow, f.g, pol_w);
            tma_load_3d_hint(st + kFfnBoxW, f.kind == 0 ? &tmWsu : &tmWu, &full[s], kc, wrow, f.g, pol_w);
            tma_load_2d(st + 2 * kFfnBoxW, f.kind == 0 ? &tmXs : &tmX, &full[s], kc, f.row0);
          } else {
            const int n = min(2, f.nkb - kb);
            mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(n) * (kFfnBoxW + kFfnBoxX));
            for (int h = 0; h < n; ++h) {
              uint8_t* sh = st + h * (kFfnBoxW + kFfnBoxX);
              const int k = kb + h;
              if (f.kind == 2) {
                const int j = k / a.sh_kb_per_j, kc = (k - j * a.sh_kb_per_j) * kFfnBK;
                tma_load_3d_hint(sh, &tmWsd, &full[s], kc, wrow, j, pol_w);
                tma_load_2d(sh + kFfnBoxW, &tmHs, &full[s], j * a.sh_k_per_j + kc, f.row0);
              } else {
                const int kc = k * kFfnBK;
                tma_load_3d_hint(sh, &tmWd, &full[s], kc, wrow, f.g, pol_w);
                tma_load_2d(sh + kFfnBoxW, &tmH, &full[s], kc, f.row0);
              }
            }
          }
          ++issued;
          if (++s == kFfnStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
    }
    if (lane == 0) {
      // no copy may still be landing in shared memory when the CTA exits
      for (int st = 0; st < kFfnStages; ++st) {
        if (issued > st) {
          const int n = (issued - 1 - st) / kFfnStages + 1;
          mbar_wait_drain(&full[st], static_cast<uint32_t>((n - 1) & 1), a.timeout_ns);
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------ MMA issuer --------------------------------
    const uint32_t idesc = idesc_bf16_f32(kFfnWB, kFfnTB);
    int s = 0, buf = 0, it = 0;
    uint32_t ph = 0, buf_ph = 0, it_ph = 0;
    bool stop = false;
    if (a.debug_wait && blockIdx.x == 0 && !mbar_wait(never, 0, 20ull * 1000 * 1000, abort_flag)) {
      ffn_record_error(a.err, abort_flag, 10);
      stop = true;
    }
    while (!stop) {
      if (!mbar_wait(&item_full[it], it_ph, a.timeout_ns, abort_flag)) {
        ffn_record_error(a.err, abort_flag, 4);
        break;
      }
      const FfnItem f = items[it];
      mbar_arrive(&item_empty[it]);
      if (++it == kFfnItems) {
        it = 0;
        it_ph ^= 1u;
      }
      if (f.kind < 0) break;
      if (!mbar_wait(&acc_empty[buf], buf_ph ^ 1u, a.timeout_ns, abort_flag)) {
        ffn_record_error(a.err, abort_flag, 5);
        break;
      }
      tc_fence_after_sync();
      const uint32_t d0 = tmem + static_cast<uint32_t>(buf * 64);
      const int per = f.kind >= 2 ? 2 : 1;
      bool ok = true;
      for (int kb = 0; kb < f.nkb; kb += per) {
        if (!mbar_wait(&full[s], ph, a.timeout_ns, abort_flag)) {
          ffn_record_error(a.err, abort_flag, 6);
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t st = smem_u32(smem + s * kFfnStage);
        if (f.kind < 2) {
          const uint64_t xd = sw128_kmajor_desc(st + 2 * kFfnBoxW);
#pragma unroll
          for (int acc = 0; acc < 2; ++acc) {
            const uint64_t wd = sw128_kmajor_desc(st + acc * kFfnBoxW);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_ss(d0 + acc * kFfnTB, wd + 2 * kk, xd + 2 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
        } else {
          const int n = min(2, f.nkb - kb);
          for (int h = 0; h < n; ++h) {
            const uint32_t sh = st + h * (kFfnBoxW + kFfnBoxX);
            const uint64_t wd = sw128_kmajor_desc(sh), xd = sw128_kmajor_desc(sh + kFfnBoxW);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_ss(d0, wd + 2 * kk, xd + 2 * kk, idesc, (kb + h > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);
        if (++s == kFfnStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      umma_commit(&acc_full[buf]);
      if (++buf == kFfnAccBufs) {
        buf = 0;
        buf_ph ^= 1u;
      }
    }
    umma_commit(teardown);
    mbar_wait_drain(teardown, 0, a.timeout_ns);
  } else if (warp >= 2) {
    // ------------------------------ epilogue ----------------------------------
    const int q = warp & 3;       // TMEM lanes 32*q .. +31
    const int r = q * 32 + lane;  // weight row of the tile = output column within the block
    int buf = 0, it = 0;
    uint32_t buf_ph = 0, it_ph = 0;
    while (true) {
      bool ok = mbar_wait(&item_full[it], it_ph, a.timeout_ns, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) ffn_record_error(a.err, abort_flag, 7);
        break;
      }
      const FfnItem f = items[it];
      __syncwarp();
      if (lane == 0) mbar_arrive(&item_empty[it]);
      if (++it == kFfnItems) {
        it = 0;
        it_ph ^= 1u;
      }
      if (f.kind < 0) break;
      ok = mbar_wait(&acc_full[buf], buf_ph, a.timeout_ns, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) ffn_record_error(a.err, abort_flag, 8);
        break;
      }
      tc_fence_after_sync();
      const bool gu = f.kind < 2;
      float v0[32], v1[32];
      const uint32_t tb = tmem + static_cast<uint32_t>(buf * 64) + (static_cast<uint32_t>(q * 32) << 16);
      ffn_tmem_ld32(tb, v0);
      if (gu) ffn_tmem_ld32(tb + kFfnTB, v1);
      tmem_ld_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);  // the accumulator is in registers: free it
      if (++buf == kFfnAccBufs) {
        buf = 0;
        buf_ph ^= 1u;
      }
      // kept short: this code runs while the weight stream fills the memory
      // system, and every instruction line it misses waits in that queue
      const int col = f.wb * kFfnWB + r;
      const bool shared = f.kind == 0 || f.kind == 2;
      const int n_limit = f.kind == 0 ? a.sh_cols : f.kind == 1 ? a.I : a.d;
      if (col < n_limit) {
        __nv_bfloat16* obase = f.kind == 0 ? a.hs : f.kind == 1 ? a.h : f.kind == 2 ? a.ys : a.y;
        const int ld = f.kind == 0 ? a.sh_cols : f.kind == 1 ? a.I : a.d;
        __nv_bfloat16* op = obase + static_cast<size_t>(f.row0) * ld + col;
        const float* rs = shared ? nullptr : a.row_scale + f.row0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (j < f.nvalid) {
            float o;
            if (gu) o = __fdividef(v0[j], 1.f + __expf(-v0[j])) * v1[j];  // SiLU(g) u
            else o = shared ? v0[j] : rs[j] * v0[j];
            *op = __float2bfloat16_rn(o);
          }
          op += ld;
        }
      }
      if (gu) {
        // this warp's rows of the tile are in H: count them for the down tiles
        fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(ready + f.ready, 1u);
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kFfnTmemCols);
  }
  // the last CTA to finish leaves the counters at zero for the next launch (all of its threads clear them)
  __shared__ uint32_t s_last;
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(ctas_done, 1u) == gridDim.x - 1 ? 1u : 0u;
  }
  __syncthreads();
  if (s_last) {
    __threadfence();
    for (int i = tid; i < kFfnMaxBlocks; i += kFfnThreads) ready[i] = 0u;
    __syncthreads();
    if (tid == 0) {
      *next_tile = 0u;
      __threadfence();
      *ctas_done = 0u;
    }
  }
}

}  // namespace fgs
