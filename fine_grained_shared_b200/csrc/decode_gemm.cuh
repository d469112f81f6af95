// decode_gemm.cuh -- steps 4 and 5 of the layer for small batches (decode):
// the expert FFNs as weight-streaming grouped GEMMs.
//
// FFN_i(u) = W_down,i (SiLU(W_gate,i u) * (W_up,i u)) for every routed expert
// i (the fine-grained experts of DeepSeekMoE, arXiv 2401.06066, Abstract and
// blog section "Fine-Grained Expert Segmentation (Section 3.1)") and for the
// always-active shared experts (blog section "Shared Expert Isolation
// (Section 3.2)").
//
// With a few dozen tokens, each expert sees a handful of rows and the layer
// is bound by reading its weights from HBM once.  So the weights are the
// MMA's 128-row operand and the tokens its N = 32 columns:
//   D[128 weight rows, 32 tokens] += W[128, 16] * X[32, 16]^T
// (tcgen05.mma, M = 128, N = 32), and every byte staged in shared memory is
// read by the MMA.  A tile is (expert, 32-token block, 128-row weight block)
// with its whole K loop; the gate/up projection stages W_gate and W_up rows
// of the same block and keeps two accumulators (SwiGLU needs both), the down
// projection one.  Tiles are weight-block major, so the token blocks of one
// weight block follow each other and re-read those weights from L2.
//
// Work is split stream-K: the k-blocks of all tiles of a space (the shared
// experts' tiles, then the routed experts' tiles, each space balanced on its
// own) are cut into equal contiguous ranges, one per CTA, so every SM streams
// the same number of weight bytes whatever the number of tiles.  A tile cut
// between CTAs is finished by the last of its contributors to arrive (a
// per-tile counter): each contributor stores its fp32 partial sums, and the
// last one adds them in k order (so the result does not depend on which CTA
// arrives last), applies the epilogue, and resets the counter.  Each of the
// four epilogue warps counts and finishes its own 32 rows of a split tile on
// its own counter, so no barrier joins the epilogue warps.
//
// One persistent CTA per SM, 192 threads:
//   warp 0      TMA producer: per 64-column k-block the weight boxes
//               [128 rows, 64] and the token box [32 rows, 64] (128-byte
//               swizzle) into a ring of kStages stages.  Weights are read
//               once, so their loads carry an L2 evict-first policy: the
//               weight stream then does not push the tokens, the partial
//               sums and the kernel's own code out of L2.
//   warp 1      allocates all 512 TMEM columns: eight accumulator buffers
//               of 64 columns, so that the MMAs run up to seven segments
//               ahead of an epilogue that is summing a split tile; one lane
//               issues the MMAs
//   warps 2-5   epilogue: thread r holds weight row r of the accumulator,
//               i.e. one output column for the tile's (up to) 32 tokens
// The gate/up kernel runs the shared experts' space before waiting on the
// router and the permutation (it reads only x and the shared weights).
#pragma once

#include "sm100.cuh"

namespace fgs {

constexpr int kDecThreads = 192;
constexpr int kDecTB = 32;    // token rows per tile (MMA N)
constexpr int kDecWB = 128;   // weight rows per tile (MMA M)
constexpr int kDecBK = 64;    // k-block: one 128-byte swizzle row of bf16
constexpr uint32_t kDecBoxW = kDecWB * kDecBK * 2;  // 16 KB
constexpr uint32_t kDecBoxX = kDecTB * kDecBK * 2;  // 4 KB
constexpr int kDecAccBufs = 8;                      // accumulator buffers of 64 columns
constexpr uint32_t kDecTmemCols = 64 * kDecAccBufs;  // all 512 columns: one CTA per SM
constexpr int kDecMinIters = 4;                     // fewest k-blocks in a CTA's range
// TMA box heights the host must encode
constexpr uint32_t kDecBoxRowsW = kDecWB;
constexpr uint32_t kDecBoxRowsX = kDecTB;

template <bool GU>
struct DecCfg;
// Ring depth: about 145 KB per SM in flight covers an SM's share of HBM
// bandwidth (1/148 of it) over the loaded latency.  Deeper rings bring no more
// bandwidth but lengthen the queue every other access of the SM waits in:
// with 216 KB (6 gate/up stages) a cold instruction fetch or a store from the
// epilogue took several microseconds, and both kernels ran 4% slower.
template <>
struct DecCfg<true> {  // gate/up: W_gate + W_up + tokens per stage
  static constexpr int kAcc = 2;
  static constexpr int kStages = 4;
};
template <>
struct DecCfg<false> {  // down: W_down + rows of H per stage
  static constexpr int kAcc = 1;
  static constexpr int kStages = 7;
};
template <bool GU>
__host__ __device__ constexpr uint32_t dec_stage_bytes() {
  return DecCfg<GU>::kAcc * kDecBoxW + kDecBoxX;
}
// fp32 partial sums of one split tile: [acc][128 rows][32 tokens]
template <bool GU>
__host__ __device__ constexpr size_t dec_partial_floats() {
  return static_cast<size_t>(DecCfg<GU>::kAcc) * kDecWB * kDecTB;
}
// per CTA and space: two partial slots (a range holds at most one tile that
// began in an earlier range and one that continues into a later range)
template <bool GU>
__host__ __device__ constexpr size_t dec_partials_bytes(int ctas) {
  return static_cast<size_t>(2) * ctas * 2 * dec_partial_floats<GU>() * 4;
}
template <bool GU>
__host__ __device__ constexpr size_t dec_smem_bytes() {
  return 1024 + static_cast<size_t>(DecCfg<GU>::kStages) * dec_stage_bytes<GU>() +
         8 * (2 * DecCfg<GU>::kStages + 2 * kDecAccBufs + 2) + 16 + 4 * (3 * 264 + 4);
}
static_assert(dec_smem_bytes<true>() <= 232448 && dec_smem_bytes<false>() <= 232448, "shared memory");
// Each CTA takes all 512 TMEM columns, so no two decode CTAs (a gate/up CTA
// and a down CTA launched early behind it included) may share an SM: one
// would wait in tcgen05.alloc until the other ends.  Shared memory keeps
// them apart (233472 bytes per SM).
static_assert(dec_smem_bytes<true>() + dec_smem_bytes<false>() > 233472 &&
                  2 * dec_smem_bytes<true>() > 233472 && 2 * dec_smem_bytes<false>() > 233472,
              "two decode CTAs would fit on one SM");

struct DecodeArgs {
  // routed experts: the expert-ordered rows of X_perm (gate/up) or H (down)
  int num_groups;              // experts; 0: no routed tiles
  const int32_t* counts;       // [G] rows of each expert
  const int32_t* row_start;    // [G + 1] first row of each expert
  int n_wb;                    // 128-row weight blocks per expert (gate/up: over I; down: over d)
  int num_kb;                  // k-blocks of a routed tile (gate/up: over d; down: over I)
  const float* row_scale;      // down: the gate g of each row of Y
  __nv_bfloat16* out;          // H (gate/up) or Y (down)
  int ld_out, n_limit;         // row stride and valid columns of out
  // shared experts: the dense rows of x (gate/up) or Hs (down)
  int sh_rows;                 // tokens; 0: no shared tiles
  int sh_n_wb;                 // gate/up: over K_s * I_s; down: over d
  int sh_J, sh_kb_per_j;       // K loop = sh_J experts x sh_kb_per_j k-blocks (gate/up: 1 x d / 64)
  int sh_k_per_j;              // down: Hs columns of one shared expert (I_s)
  __nv_bfloat16* sh_out;       // Hs (gate/up) or Ys (down)
  int sh_ld_out, sh_n_limit;
  // stream-K scratch (zero counters between launches; each last contributor resets its tile's)
  float* partials;             // dec_partials_bytes(gridDim.x)
  uint32_t* tile_ctr;          // [4 x (shared tiles + routed tiles)]: one counter per quarter of a tile
  uint32_t* err;
  uint64_t timeout_ns;
};

// Contiguous ranges of a space's `total` k-blocks over `workers` CTAs: range
// c is [bound(c), bound(c + 1)).  Plain: equal ranges.  With lead tiles
// (lead > 0): the first `lead` CTAs each also run one whole tile of lead_kbt
// k-blocks of another space, and the ranges of this space are shifted so
// that every CTA's total comes out equal:
//   bound(c) = max(0, floor(c (total + lead lead_kbt) / workers) - min(c, lead) lead_kbt),
// which is non-decreasing and reaches total at c = workers.
struct DecSpace {
  long long total;
  int workers, kbt;  // kbt: k-blocks of every tile of the space
  int lead, lead_kbt;
  __device__ __forceinline__ long long bound(int c) const {
    const long long all = total + static_cast<long long>(lead) * lead_kbt;
    const long long b = static_cast<long long>(c) * all / workers - static_cast<long long>(min(c, lead)) * lead_kbt;
    return b < 0 ? 0 : b;
  }
  // the CTA whose range holds k-block x: the largest c with bound(c) <= x
  // (empty ranges hold none)
  __device__ __forceinline__ int cta_of(long long x) const {
    int lo = 0, hi = workers;  // bound(lo) <= x < bound(hi), bound(workers) = total
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (bound(mid) <= x) lo = mid;
      else hi = mid;
    }
    return lo;
  }
};

__device__ __forceinline__ DecSpace dec_space(long long tiles, int kbt, int ctas) {
  DecSpace s;
  s.total = tiles * kbt;
  s.kbt = kbt > 0 ? kbt : 1;
  s.lead = 0;
  s.lead_kbt = 0;
  const long long w = s.total / kDecMinIters;
  s.workers = static_cast<int>(w < 1 ? 1 : w > ctas ? ctas : w);
  if (s.total == 0) s.workers = 1;
  return s;
}

struct DecTile {
  int g;        // routed: expert; shared: 0
  int wb;       // weight block
  int row0;     // first token row (of X_perm / H, or of x / Hs)
  int nvalid;   // token rows of the block that exist
};

// routed tile t: weight-block major within an expert
__device__ __forceinline__ DecTile dec_routed_tile(long long t, const int32_t* s_tbs, const int32_t* s_rows,
                                                   const int32_t* s_cnt, int G, int n_wb) {
  int lo = 0, hi = G;  // largest g with s_tbs[g] * n_wb <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (static_cast<long long>(s_tbs[mid]) * n_wb <= t) lo = mid;
    else hi = mid;
  }
  const int ntb = s_tbs[lo + 1] - s_tbs[lo];
  const int local = static_cast<int>(t - static_cast<long long>(s_tbs[lo]) * n_wb);
  DecTile d;
  d.g = lo;
  d.wb = local / ntb;
  const int tb = local - d.wb * ntb;
  d.row0 = s_rows[lo] + tb * kDecTB;
  d.nvalid = min(kDecTB, s_cnt[lo] - tb * kDecTB);
  return d;
}

__device__ __forceinline__ DecTile dec_shared_tile(long long t, int sh_rows) {
  const int ntb = (sh_rows + kDecTB - 1) / kDecTB;
  DecTile d;
  d.g = 0;
  d.wb = static_cast<int>(t / ntb);
  const int tb = static_cast<int>(t - static_cast<long long>(d.wb) * ntb);
  d.row0 = tb * kDecTB;
  d.nvalid = min(kDecTB, sh_rows - tb * kDecTB);
  return d;
}

// Walks one CTA's range of a space as segments (tile, k-blocks [k0, k1)) in
// k order: its head (the end of a tile an earlier CTA began), the whole tiles,
// then its tail (the start of a tile a later CTA finishes).  Whichever CTA
// counts a cut tile's last part sums the parts.  (Taking the tail before the
// whole tiles, so that its sum happens earlier, measured 3-5% slower on the
// gate/up GEMM of the 16B decode layer.)
struct DecWalk {
  long long lo[3], hi[3], x;
  int n, i, kbt;
  __device__ __forceinline__ bool next(long long& tile, int& k0, int& k1) {
    while (i < n) {
      if (x < hi[i]) {
        tile = x / kbt;
        k0 = static_cast<int>(x - tile * kbt);
        const long long rem = hi[i] - x;
        k1 = static_cast<int>(k0 + rem < kbt ? k0 + rem : kbt);
        x = tile * kbt + k1;
        return true;
      }
      if (++i < n) x = lo[i];
    }
    return false;
  }
};

// The walk of [x0, x1) in tiles of kbt k-blocks.
__device__ __forceinline__ DecWalk dec_walk_range(long long x0, long long x1, int kbt) {
  DecWalk w;
  w.kbt = kbt;
  w.n = 0;
  w.i = 0;
  if (x0 < x1) {
    const long long b0 = (x0 + kbt - 1) / kbt * kbt;  // first tile boundary at or after x0
    const long long b1 = x1 / kbt * kbt;              // last tile boundary at or before x1
    if (b0 > b1) {  // inside one tile
      w.lo[0] = x0;
      w.hi[0] = x1;
      w.n = 1;
    } else {
      if (x0 < b0) { w.lo[w.n] = x0; w.hi[w.n] = b0; ++w.n; }  // head
      if (b0 < b1) { w.lo[w.n] = b0; w.hi[w.n] = b1; ++w.n; }  // whole tiles
      if (b1 < x1) { w.lo[w.n] = b1; w.hi[w.n] = x1; ++w.n; }  // tail
    }
  }
  w.x = w.n ? w.lo[0] : 0;
  return w;
}

__device__ __forceinline__ DecWalk dec_walk(const DecSpace& s, int c) {
  if (c >= s.workers || s.total == 0) return dec_walk_range(0, 0, s.kbt);
  return dec_walk_range(s.bound(c), s.bound(c + 1), s.kbt);
}

__device__ __forceinline__ void dec_record_error(uint32_t* err, volatile int* abort, uint32_t site) {
  *abort = 1;
  atomicOr(err, kErrTimeout | (1u << (kErrSiteShift + site)));
}

// 32 lanes x 32 columns of 32-bit TMEM cells
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[16];
  tmem_ld16(taddr, r);
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
  tmem_ld16(taddr + 16, r);
#pragma unroll
  for (int j = 0; j < 16; ++j) v[16 + j] = __uint_as_float(r[j]);
}

// tmW0 / tmW1: the routed experts' weights as [G][rows][k] with a 128-row box
// (gate/up: W_gate and W_up; down: W_down, tmW1 unused); tmX: X_perm or H
// with a 32-row box.  tmWs0 / tmWs1 / tmXs: the shared experts' (gate/up:
// W_gate,s and W_up,s as [1][K_s * I_s][d] and x; down: W_down,s as
// [K_s][d][I_s] and Hs).  Maps of an absent part are never read.
template <bool GU>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_gemm_kernel(const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmW1,
                       const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWs0,
                       const __grid_constant__ CUtensorMap tmWs1, const __grid_constant__ CUtensorMap tmXs,
                       DecodeArgs a) {
  constexpr int S = DecCfg<GU>::kStages;
  constexpr int NA = DecCfg<GU>::kAcc;
  constexpr uint32_t kStage = dec_stage_bytes<GU>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * kStage);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;                // [kDecAccBufs]
  uint64_t* acc_empty = acc_full + kDecAccBufs;  // [kDecAccBufs]
  uint64_t* tables = acc_empty + kDecAccBufs;    // the routed tables are in shared memory
  uint64_t* teardown = tables + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(teardown + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_tbs = reinterpret_cast<int32_t*>(tmem_slot + 4);  // [264] prefix of 32-token blocks
  int32_t* s_rows = s_tbs + 264;                                // [264]
  int32_t* s_cnt = s_rows + 264;                                // [264]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.num_groups;
  const int ctas = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const long long sh_tiles =
      a.sh_rows > 0 ? static_cast<long long>((a.sh_rows + kDecTB - 1) / kDecTB) * a.sh_n_wb : 0;
  // The shared experts' tiles need neither the router nor the permutation
  // (they run before the grid dependency wait).  When they fit one per CTA
  // the first sh_tiles CTAs each run one whole (no tile is cut, so no partial
  // sums are summed later), and the routed ranges are shifted to even out
  // every CTA's k-blocks; otherwise the shared space is cut like the routed
  // one.  (Cutting every shared tile between ~7 CTAs left the CTAs that sum
  // the parts up to 50 us behind the rest on the 16B decode layer.)
  const int sh_kbt = a.sh_J * a.sh_kb_per_j;
  const bool sh_whole = sh_tiles > 0 && sh_tiles <= ctas;
  const DecSpace sp0 = dec_space(sh_whole ? 0 : sh_tiles, sh_kbt, ctas);

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < kDecAccBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);  // one arrive per epilogue warp
    }
    mbar_init(tables, 1);
    mbar_init(teardown, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kDecTmemCols);
    tmem_relinquish();
  }
  if (!GU) pdl_wait();  // H, Hs and the router's tables come from earlier kernels
  pdl_launch_dependents();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  // the routed space needs the router's counts: the producer warp loads them
  // after the grid dependency wait and publishes them on `tables`
  auto routed_space = [&]() {
    const long long tiles = G ? static_cast<long long>(s_tbs[G]) * a.n_wb : 0;
    DecSpace sp = dec_space(tiles, a.num_kb, ctas);
    // shifted ranges only when every CTA's range keeps at least kDecMinIters
    // k-blocks (a split tile's parts must come from consecutive CTAs, none
    // empty); a small batch keeps the plain ranges and the lead CTAs' extra tile
    const long long all = tiles * a.num_kb + sh_tiles * sh_kbt;
    if (sh_whole && all / ctas >= sh_kbt + kDecMinIters) {
      sp.workers = ctas;
      sp.lead = static_cast<int>(sh_tiles);
      sp.lead_kbt = sh_kbt;
    }
    return sp;
  };
  // the shared segments of CTA c: one whole tile, or its cut range
  auto shared_walk = [&]() {
    if (sh_whole) {
      const long long x0 = c < sh_tiles ? static_cast<long long>(c) * sh_kbt : 0;
      return dec_walk_range(x0, c < sh_tiles ? x0 + sh_kbt : 0, sh_kbt);
    }
    return dec_walk(sp0, c);
  };
  // a whole shared tile is never cut: the space's k-block count of a tile
  const DecSpace sp0w = [&]() {
    DecSpace t = sp0;
    if (sh_whole) t.kbt = sh_kbt;
    return t;
  }();

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    int s = 0, issued = 0;
    const uint64_t pol_w = l2_policy_evict_first();
    uint32_t ph = 0;
    bool stop = false;
    auto load_segment = [&](bool shared, const DecTile& t, int k0, int k1) {
      for (int kb = k0; kb < k1 && !stop; ++kb) {
        if (!mbar_wait(&empty[s], ph ^ 1u, a.timeout_ns, abort_flag)) {
          dec_record_error(a.err, abort_flag, 3);
          stop = true;
          break;
        }
        uint8_t* st = smem + s * kStage;
        mbar_arrive_expect_tx(&full[s], kStage);
        const int wrow = t.wb * kDecWB;
        if (GU) {
          const int kc = kb * kDecBK;
          tma_load_3d_hint(st, shared ? &tmWs0 : &tmW0, &full[s], kc, wrow, t.g, pol_w);
          tma_load_3d_hint(st + kDecBoxW, shared ? &tmWs1 : &tmW1, &full[s], kc, wrow, t.g, pol_w);
          tma_load_2d(st + 2 * kDecBoxW, shared ? &tmXs : &tmX, &full[s], kc, t.row0);
        } else if (shared) {
          const int j = kb / a.sh_kb_per_j, kc = (kb - j * a.sh_kb_per_j) * kDecBK;
          tma_load_3d_hint(st, &tmWs0, &full[s], kc, wrow, j, pol_w);
          tma_load_2d(st + kDecBoxW, &tmXs, &full[s], j * a.sh_k_per_j + kc, t.row0);
        } else {
          const int kc = kb * kDecBK;
          tma_load_3d_hint(st, &tmW0, &full[s], kc, wrow, t.g, pol_w);
          tma_load_2d(st + kDecBoxW, &tmX, &full[s], kc, t.row0);
        }
        ++issued;
        if (++s == S) {
          s = 0;
          ph ^= 1u;
        }
      }
    };
    if (lane == 0) {
      if (sh_tiles) {
        tma_prefetch_desc(&tmWs0);
        if (GU) tma_prefetch_desc(&tmWs1);
        tma_prefetch_desc(&tmXs);
      }
      if (G) {
        tma_prefetch_desc(&tmW0);
        if (GU) tma_prefetch_desc(&tmW1);
        tma_prefetch_desc(&tmX);
      }
      DecWalk w = shared_walk();
      long long tile;
      int k0, k1;
      while (!stop && w.next(tile, k0, k1)) load_segment(true, dec_shared_tile(tile, a.sh_rows), k0, k1);
    }
    if (GU) pdl_wait();  // the router's tables and the permuted rows are complete from here
    // 32-token blocks of each expert, prefix-summed (a warp scan of per-lane sums)
    int run = 0, loc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int g = lane * 8 + i;
      const int cnt = g < G ? a.counts[g] : 0;
      loc[i] = (cnt + kDecTB - 1) / kDecTB;
      if (g < G) {
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
      if (g <= G) s_tbs[g] = ex;
      ex += loc[i];
    }
    if (lane == 31 && G == 256) s_tbs[256] = incl;  // the total, past the last lane's experts
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(tables);
      const DecSpace sp1 = routed_space();
      DecWalk w = dec_walk(sp1, c);
      long long tile;
      int k0, k1;
      while (!stop && w.next(tile, k0, k1))
        load_segment(false, dec_routed_tile(tile, s_tbs, s_rows, s_cnt, G, a.n_wb), k0, k1);
      // no copy may still be landing in shared memory when the CTA exits
      for (int st = 0; st < S; ++st) {
        if (issued > st) {
          const int n = (issued - 1 - st) / S + 1;
          mbar_wait_drain(&full[st], static_cast<uint32_t>((n - 1) & 1), a.timeout_ns);
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------ MMA issuer --------------------------------
    const uint32_t idesc = idesc_bf16_f32(kDecWB, kDecTB);
    int s = 0, buf = 0;
    uint32_t ph = 0, buf_ph = 0;
    bool stop = false;
    auto mma_segment = [&](int k0, int k1) {
      if (!mbar_wait(&acc_empty[buf], buf_ph ^ 1u, a.timeout_ns, abort_flag)) {
        dec_record_error(a.err, abort_flag, 5);
        stop = true;
        return;
      }
      tc_fence_after_sync();
      const uint32_t d0 = tmem + static_cast<uint32_t>(buf * 64);
      for (int kb = k0; kb < k1; ++kb) {
        if (!mbar_wait(&full[s], ph, a.timeout_ns, abort_flag)) {
          dec_record_error(a.err, abort_flag, 6);
          stop = true;
          return;
        }
        tc_fence_after_sync();
        const uint32_t st = smem_u32(smem + s * kStage);
        const uint64_t xd = sw128_kmajor_desc(st + NA * kDecBoxW);
#pragma unroll
        for (int acc = 0; acc < NA; ++acc) {
          const uint64_t wd = sw128_kmajor_desc(st + acc * kDecBoxW);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_ss(d0 + acc * kDecTB, wd + 2 * kk, xd + 2 * kk, idesc, (kb > k0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
        if (++s == S) {
          s = 0;
          ph ^= 1u;
        }
      }
      umma_commit(&acc_full[buf]);
      if (++buf == kDecAccBufs) {
        buf = 0;
        buf_ph ^= 1u;
      }
    };
    {
      DecWalk w = shared_walk();
      long long tile;
      int k0, k1;
      while (!stop && w.next(tile, k0, k1)) mma_segment(k0, k1);
    }
    if (!stop && !mbar_wait(tables, 0, a.timeout_ns, abort_flag)) {
      dec_record_error(a.err, abort_flag, 11);
      stop = true;
    }
    if (!stop) {
      const DecSpace sp1 = routed_space();
      DecWalk w = dec_walk(sp1, c);
      long long tile;
      int k0, k1;
      while (!stop && w.next(tile, k0, k1)) mma_segment(k0, k1);
    }
    umma_commit(teardown);
    mbar_wait_drain(teardown, 0, a.timeout_ns);
  } else if (warp >= 2) {
    // ------------------------------ epilogue ----------------------------------
    const int q = warp & 3;    // TMEM lanes 32*q .. +31
    const int r = q * 32 + lane;  // weight row of the tile = output column within the block
    int buf = 0;
    uint32_t buf_ph = 0;
    bool stop = false;
    auto epilogue = [&](int space, const DecSpace& sp, long long tile, int k0, int k1, bool shared,
                        const DecTile& t) {
      bool ok = mbar_wait(&acc_full[buf], buf_ph, a.timeout_ns, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) dec_record_error(a.err, abort_flag, 7);
        stop = true;
        return;
      }
      tc_fence_after_sync();
      float v[NA][32];
      const uint32_t tb = tmem + static_cast<uint32_t>(buf * 64) + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
      for (int acc = 0; acc < NA; ++acc) tmem_ld32(tb + acc * kDecTB, v[acc]);
      tmem_ld_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);  // the accumulator is in registers: free it
      if (++buf == kDecAccBufs) {
        buf = 0;
        buf_ph ^= 1u;
      }
      const int nv4 = (t.nvalid + 3) >> 2;  // 4-token groups holding the valid tokens
      if (k0 != 0 || k1 != sp.kbt) {
        // a tile cut between CTAs: each warp stores its 32 rows of this part, counts them on
        // the tile's counter for its quarter, and the warp that counts the last part of the
        // quarter sums the parts (no barrier across warps, so a warp that stops waits on no one)
        const long long t0 = tile * sp.kbt;
        const int cf = sp.cta_of(t0), cl = sp.cta_of(t0 + sp.kbt - 1);
        auto slot_ptr = [&](int cta) {
          const int slot = cta == cf ? 1 : 0;  // the first part is its range's tail; later ones heads
          return a.partials +
                 ((static_cast<size_t>(space) * ctas + cta) * 2 + slot) * dec_partial_floats<GU>();
        };
        float* mine = slot_ptr(c);
#pragma unroll
        for (int acc = 0; acc < NA; ++acc)
#pragma unroll
          for (int j4 = 0; j4 < 8; ++j4)
            if (j4 < nv4)
              *reinterpret_cast<float4*>(mine + (acc * kDecWB + r) * kDecTB + 4 * j4) =
                  make_float4(v[acc][4 * j4], v[acc][4 * j4 + 1], v[acc][4 * j4 + 2], v[acc][4 * j4 + 3]);
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          const long long ctr = (space ? (sh_tiles + tile) : tile) * 4 + q;
          const uint32_t old = atomicAdd(a.tile_ctr + ctr, 1u);
          last = old == static_cast<uint32_t>(cl - cf);
          if (last) a.tile_ctr[ctr] = 0u;  // every part has counted itself: ready for the next launch
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) return;
        __threadfence();
        // the sum of the parts in k order
#pragma unroll
        for (int acc = 0; acc < NA; ++acc)
#pragma unroll
          for (int j = 0; j < 32; ++j) v[acc][j] = 0.f;
        for (int cta = cf; cta <= cl; ++cta) {
          const float* part = slot_ptr(cta);
#pragma unroll
          for (int acc = 0; acc < NA; ++acc)
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4)
              if (j4 < nv4) {
                const float4 p =
                    __ldcg(reinterpret_cast<const float4*>(part + (acc * kDecWB + r) * kDecTB + 4 * j4));
                v[acc][4 * j4] += p.x;
                v[acc][4 * j4 + 1] += p.y;
                v[acc][4 * j4 + 2] += p.z;
                v[acc][4 * j4 + 3] += p.w;
              }
        }
      }
      // epilogue of a finished tile: column col of each valid token's row
      const int col = t.wb * kDecWB + r;
      const int n_limit = shared ? a.sh_n_limit : a.n_limit;
      if (col >= n_limit) return;
      __nv_bfloat16* obase = shared ? a.sh_out : a.out;
      const int ld = shared ? a.sh_ld_out : a.ld_out;
      // kept short: this code first runs while the weight stream fills the
      // memory system, and every instruction line it misses waits in that queue
      __nv_bfloat16* op = obase + static_cast<size_t>(t.row0) * ld + col;
      const float* rs = shared ? nullptr : a.row_scale + t.row0;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j < t.nvalid) {
          float o;
          if (GU) {
            const float g = v[0][j], u = v[1][j];
            o = __fdividef(g, 1.f + __expf(-g)) * u;  // SiLU(g) u
          } else {
            o = shared ? v[0][j] : rs[j] * v[0][j];
          }
          *op = __float2bfloat16_rn(o);
        }
        op += ld;
      }
    };
    {
      DecWalk w = shared_walk();
      long long tile;
      int k0, k1;
      while (!stop && w.next(tile, k0, k1)) epilogue(0, sp0w, tile, k0, k1, true, dec_shared_tile(tile, a.sh_rows));
    }
    bool okt = stop ? false : mbar_wait(tables, 0, a.timeout_ns, abort_flag);
    okt = __all_sync(0xffffffffu, okt);
    if (!okt && !stop) {
      if (lane == 0) dec_record_error(a.err, abort_flag, 12);
      stop = true;
    }
    if (!stop) {
      const DecSpace sp1 = routed_space();
      DecWalk w = dec_walk(sp1, c);
      long long tile;
      int k0, k1;
      while (!stop && w.next(tile, k0, k1))
        epilogue(1, sp1, tile, k0, k1, false, dec_routed_tile(tile, s_tbs, s_rows, s_cnt, G, a.n_wb));
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kDecTmemCols);
  }
}

}  // namespace fgs
