// down_gemm.cuh -- step 5 of the layer: the expert FFNs' second half,
// FFN_i = H_i W_down,i^T, as grouped GEMMs on CTA pairs of the 5th-generation
// tensor cores, with the gate scale fused into the epilogue.
//
// FFN_i(u) = W_down,i (SiLU(W_gate,i u) * (W_up,i u)) for every routed expert
// i (the fine-grained experts of DeepSeekMoE, arXiv 2401.06066, Abstract and
// blog section "Fine-Grained Expert Segmentation (Section 3.1)") and for the
// always-active shared experts (blog section "Shared Expert Isolation
// (Section 3.2)"); h_t = u_t + sum_j FFN^shared_j(u_t) + sum_k g_{t,k} FFN(u_t).
//
// One persistent kernel template launched as CTA pairs (clusters of 2), one
// CTA per SM, 192 threads per CTA.  A pair computes a 256 x 256 output tile
// with the 2-SM MMA (tcgen05.mma.cta_group::2, M = 256, N = 256, K = 16):
// each CTA stages its own 128 rows of A and its own 128 rows of B, which
// halves the shared-memory operand traffic per FLOP of a 1-SM 128 x 256 tile.
//   warp 0      TMA producer (both CTAs): A [128 rows, 64] and B [128 rows, 64]
//               per k-block into a 6-stage ring (128-byte swizzle); the copies
//               of both CTAs complete on the even CTA's full barrier
//   warp 1      allocates 512 TMEM columns for the pair; in the even CTA one
//               lane issues the pair MMAs into one of two 256-column fp32
//               accumulators (the epilogue of tile i overlaps the MMAs of
//               tile i + 1) and multicasts its commits to both CTAs
//   warps 2-5   epilogue (both CTAs); warp w reads TMEM lanes 32*(w%4) .. +31
//               (one output row per thread) and releases the accumulator on
//               the even CTA's barrier
// One launch covers both kinds of expert.  Its tiles are (part, group,
// 256-row m-tile, 256-column n-tile): first the shared experts' tiles over
// the rows of Hs, whose K loop runs over (shared expert j, 64-column block)
// with a 3-D map of W_down,s [K_s][d][I_s] so that one accumulator sums the
// shared experts, then one group per routed expert (its rows are read from
// device-side offsets written by the router, so the host never synchronises;
// every expert's rows start on a 256-row boundary).  The longer shared tiles
// go first so that they do not make the tail.  Pairs take tiles in a static
// round-robin order.
//
// Epilogue: Y[row, n0 + c] = g[row] * acc[c] (bf16) for routed tiles and
// Ys[row, n0 + c] = acc[c] for shared ones.  The layer's final k-ordered sum
// runs in combine_kernel, which streams whole rows (permute.cuh): summing in
// this epilogue, each output chunk by the last of its K + 1 producers to
// arrive, left the epilogue warps waiting on scattered row reads longer than
// the next tile's MMAs (16B prefill: down 0.92 ms against 0.56 + 0.145 ms for
// down and combine).
#pragma once

#include "sm100.cuh"

namespace fgs {

constexpr int kGemmThreads = 192;
constexpr int kGemmStages = 6;
constexpr int kGemmBM = 256;      // rows of a pair tile (128 per CTA)
constexpr int kCtaRows = 128;
constexpr int kGemmBN = 256;      // MMA N
constexpr int kGemmBK = 64;
constexpr uint32_t kStageA = kCtaRows * kGemmBK * 2;        // 16 KB: this CTA's A rows
constexpr uint32_t kStageB = (kGemmBN / 2) * kGemmBK * 2;   // 16 KB: this CTA's half of B
constexpr uint32_t kTmemCols = 512;
// TMA box heights the host must encode: A maps and B maps (one CTA's share)
constexpr uint32_t kBoxRowsA = kCtaRows;
constexpr uint32_t kBoxRowsB = kGemmBN / 2;
static_assert(kStageA == kBoxRowsA * kGemmBK * 2 && kStageB == kBoxRowsB * kGemmBK * 2, "stage = one TMA box");


// Shared-memory matrix descriptor of an MN-major operand in the 128-byte swizzle: the tile is stored as
// chunks of 64 MN elements (128 bytes) x its K rows, chunk after chunk `lbo` bytes apart, each chunk's
// rows 128 bytes apart with the 16-byte units of row r XOR-ed with r % 8 (the layout a TMA box of
// 64 MN elements x K rows writes); groups of 8 K rows are 1024 bytes apart.  A step of 16 K rows
// moves the start address by 2048 bytes.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t saddr, uint32_t lbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

struct GemmArgs {
  // routed experts (grouped rows of H; tiles after the shared ones)
  int num_groups;              // experts; 0: no routed tiles
  const int32_t* mtile_start;  // [num_groups + 1] prefix sum of ceil(count / 256)
  const int32_t* row_start;    // [num_groups + 1]
  int num_kb;                  // 64-wide k-blocks over I
  const float* row_scale;      // g of each row of Y, or nullptr: 1
  __nv_bfloat16* out;          // Y
  // shared experts (dense rows of Hs; their tiles come first)
  int sh_rows;                 // tokens; 0: no shared tiles
  int sh_num_kb;               // 64-wide k-blocks over I_s
  int sh_J;                    // shared experts summed into one accumulator
  int sh_k_per_j;              // Hs columns per shared expert (I_s)
  __nv_bfloat16* sh_out;       // Ys
  // both parts
  int n_tiles;                 // 256-column output tiles (over d)
  int n_limit;                 // valid output columns (d)
  int ld_out;
  uint32_t* err;
  uint64_t timeout_ns;
  int debug_wait;              // CTA 0 waits on a barrier nothing arrives on
  // weight-gradient mode (kg_groups > 0; the parts above unused): group g multiplies rows
  // [g * kg_a_row_step, + kg_M) of A by the rows of B (third coordinate g * kg_bz_step), both
  // K-major, over the K range [kg_k_start[g], + kg_k_count[g]) (zero beyond the count: the
  // operands hold zeros there); fp32 output [kg_M rows][n_limit] per group, rows >= kg_split of a
  // group into kg_out2
  int kg_groups;
  const int32_t* kg_k_start;   // [groups], multiples of 8
  const int32_t* kg_k_count;   // [groups]
  int kg_m_tiles;              // 256-row tiles of a group's kg_M rows
  int kg_M;
  int kg_a_row_step;
  int kg_bz_step;
  int kg_split;
  int kg_ld;                   // output row stride (>= n_limit, a multiple of 16)
  // bit 0: A MN-major, bit 1: B MN-major -- a row-major [K rows][MN columns] buffer read through a
  // 2-D map with 64 x 64 boxes, two per operand and stage; group g's A columns start at
  // g * kg_a_row_step and its B columns at g * kg_b_col_step (with kg_bz_step set); a clear bit: that
  // operand K-major as described above
  int kg_mn;
  int kg_b_col_step;
  float* kg_out;               // [groups][kg_split][kg_ld]
  float* kg_out2;              // [groups][kg_M - kg_split][kg_ld]
};

__host__ __device__ constexpr size_t gemm_smem_bytes() {
  return 1024 + static_cast<size_t>(kGemmStages) * (kStageA + kStageB) + 8 * (2 * kGemmStages + 4 + 2) + 16 +
         4 * 2 * 264;
}

struct TileCoord {
  int shared;  // 1: a shared-expert tile over the rows of Hs
  int g, m_tile, n_tile, row0;
};

// tiles [0, sh_tiles) are the shared experts' (m-tile major); the rest are
// the routed experts', expert by expert
__device__ __forceinline__ TileCoord decode_tile(int tile, int sh_tiles, const int32_t* s_mts,
                                                 const int32_t* s_rows, int G, int n_tiles) {
  TileCoord c;
  if (tile < sh_tiles) {
    c.shared = 1;
    c.g = 0;
    c.m_tile = tile / n_tiles;
    c.n_tile = tile - c.m_tile * n_tiles;
    c.row0 = c.m_tile * kGemmBM;
    return c;
  }
  tile -= sh_tiles;
  // largest g with s_mts[g] * n_tiles <= tile (empty groups share a start)
  int lo = 0, hi = G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_mts[mid] * n_tiles <= tile) lo = mid;
    else hi = mid;
  }
  c.shared = 0;
  c.g = lo;
  const int local = tile - s_mts[lo] * n_tiles;
  c.m_tile = local / n_tiles;
  c.n_tile = local - c.m_tile * n_tiles;
  c.row0 = s_rows[lo] + c.m_tile * kGemmBM;
  return c;
}

// Sets the error bit and the abort flags of both CTAs of the pair (the peer
// is alive until the final cluster barrier, so its shared memory is valid).
__device__ __forceinline__ void pair_record_error(uint32_t* err, volatile int* abort, uint32_t rank, uint32_t site) {
  *abort = 1;
  const uint32_t peer = mapa_shared(smem_u32(const_cast<int*>(abort)), rank ^ 1u);
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer), "r"(1) : "memory");
  atomicOr(err, kErrTimeout | (1u << (kErrSiteShift + site)));
}

// tmA: H rows; tmB: W_down as [experts][d][I].  tmAs: Hs rows; tmBs: the
// shared experts' W_down as [K_s][d][I_s].  Maps of an absent part are never
// read.
__global__ void __launch_bounds__(kGemmThreads, 1)
    down_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmAs, const __grid_constant__ CUtensorMap tmBs, GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kGemmStages * kStageA;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kGemmStages * kStageB);  // [S], used in the even CTA
  uint64_t* empty = full + kGemmStages;                                         // [S], each CTA
  uint64_t* acc_full = empty + kGemmStages;                                     // [2], each CTA
  uint64_t* acc_empty = acc_full + 2;                                           // [2], used in the even CTA
  uint64_t* never = acc_empty + 2;
  uint64_t* teardown = never + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(teardown + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_mts = reinterpret_cast<int32_t*>(tmem_slot + 4);  // [264]
  int32_t* s_rows = s_mts + 264;                                // [264]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;

  const int G = a.num_groups;
  const int KG = a.kg_groups;
  const int kg_per_group = a.kg_m_tiles * a.n_tiles;
  const int sh_tiles = a.sh_rows > 0 ? (a.sh_rows + kGemmBM - 1) / kGemmBM * a.n_tiles : 0;
  if (tid == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 2 * 4);  // one arrive per epilogue warp of both CTAs
    }
    mbar_init(never, 1);
    mbar_init(teardown, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  pdl_wait();  // H, Hs and the router's tables are complete from here
  pdl_launch_dependents();
  if (KG) {  // weight-gradient mode: s_mts = the groups' K counts, s_rows = their K starts
    for (int i = tid; i < KG; i += kGemmThreads) {
      s_mts[i] = a.kg_k_count[i];
      s_rows[i] = a.kg_k_start[i];
    }
  } else {
    for (int i = tid; i <= G; i += kGemmThreads) {
      s_mts[i] = G ? a.mtile_start[i] : 0;
      s_rows[i] = G ? a.row_start[i] : 0;
    }
  }
  tc_fence_before_sync();
  cluster_sync();  // both CTAs' barriers exist before any copy or arrive targets them
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int total_tiles = KG ? KG * kg_per_group : sh_tiles + s_mts[G] * a.n_tiles;
  const uint32_t full_lead = mapa_shared(smem_u32(full), 0);         // the even CTA's full[0]
  const uint32_t acc_empty_lead = mapa_shared(smem_u32(acc_empty), 0);
  bool aborted = false;

  if (warp == 0 && lane == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (G) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
    }
    if (sh_tiles) {
      tma_prefetch_desc(&tmAs);
      tma_prefetch_desc(&tmBs);
    }
    int s = 0, issued = 0;
    uint32_t ph = 0;
    for (int tile = pair; tile < total_tiles && !aborted; tile += num_pairs) {
      if (KG) {
        const int g = tile / kg_per_group, local = tile - g * kg_per_group;
        const int mt = local / a.n_tiles, nt = local - mt * a.n_tiles;
        const int arow = g * a.kg_a_row_step + mt * kGemmBM + static_cast<int>(rank) * kCtaRows;
        const int brow = ((a.kg_mn & 2) && a.kg_bz_step ? g * a.kg_b_col_step : 0) + nt * kGemmBN +
                         static_cast<int>(rank) * (kGemmBN / 2);
        const int bz = a.kg_bz_step ? g : 0;
        const int nkb = (s_mts[g] + kGemmBK - 1) / kGemmBK;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, a.timeout_ns, abort_flag)) {
            pair_record_error(a.err, abort_flag, rank, 3);
            aborted = true;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * (kStageA + kStageB));
          const int kc = s_rows[g] + kb * kGemmBK;
          const uint32_t fb = full_lead + 8u * static_cast<uint32_t>(s);
          // MN-major: x = the MN column, y = the K row, two 64-column boxes per operand
          if (a.kg_mn & 1) {
            tma_load_2d_pair(sA + s * kStageA, &tmA, fb, arow, kc);
            tma_load_2d_pair(sA + s * kStageA + kStageA / 2, &tmA, fb, arow + 64, kc);
          } else {
            tma_load_2d_pair(sA + s * kStageA, &tmA, fb, kc, arow);
          }
          if (a.kg_mn & 2) {
            tma_load_2d_pair(sB + s * kStageB, &tmB, fb, brow, kc);
            tma_load_2d_pair(sB + s * kStageB + kStageB / 2, &tmB, fb, brow + 64, kc);
          } else {
            tma_load_3d_pair(sB + s * kStageB, &tmB, fb, kc, brow, bz);
          }
          ++issued;
          if (++s == kGemmStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        continue;
      }
      const TileCoord c = decode_tile(tile, sh_tiles, s_mts, s_rows, G, a.n_tiles);
      const int row0 = c.row0 + static_cast<int>(rank) * kCtaRows;
      // each CTA stages its half of the tile's 256 output columns of W_down
      const int brow = c.n_tile * kGemmBN + static_cast<int>(rank) * (kGemmBN / 2);
      const CUtensorMap* mA = c.shared ? &tmAs : &tmA;
      const CUtensorMap* mB = c.shared ? &tmBs : &tmB;
      const int J = c.shared ? a.sh_J : 1;
      const int num_kb = c.shared ? a.sh_num_kb : a.num_kb;
      for (int j = 0; j < J && !aborted; ++j) {
        // shared: sub-expert j of the one dense group; routed: expert g
        const int bz = c.shared ? j : c.g;
        const int k0 = c.shared ? j * a.sh_k_per_j : 0;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, a.timeout_ns, abort_flag)) {
            pair_record_error(a.err, abort_flag, rank, 3);
            aborted = true;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * (kStageA + kStageB));
          const int kc = kb * kGemmBK;
          const uint32_t fb = full_lead + 8u * static_cast<uint32_t>(s);
          tma_load_2d_pair(sA + s * kStageA, mA, fb, k0 + kc, row0);
          tma_load_3d_pair(sB + s * kStageB, mB, fb, kc, brow, bz);
          ++issued;
          if (++s == kGemmStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
    if (leader) {
      // every copy of the pair lands on the even CTA's barriers: wait for the
      // last phase issued on each stage before the pair may exit
      for (int st = 0; st < kGemmStages; ++st) {
        if (issued > st) {
          const int n = (issued - 1 - st) / kGemmStages + 1;
          mbar_wait_drain(&full[st], static_cast<uint32_t>((n - 1) & 1), a.timeout_ns);
        }
      }
    }
  } else if (warp == 1 && lane == 0 && leader) {
    // ------------------------- MMA issuer (even CTA) --------------------------
    // MN-major operands (per-group mode): bits 15 (A) and 16 (B) of the instruction descriptor
    const bool mn_a = KG && (a.kg_mn & 1), mn_b = KG && (a.kg_mn & 2);
    const uint32_t idesc = idesc_bf16_f32(kGemmBM, kGemmBN) | (mn_a ? 1u << 15 : 0u) | (mn_b ? 1u << 16 : 0u);
    int s = 0, acc = 0;
    uint32_t ph = 0, acc_ph = 0;
    if (a.debug_wait && blockIdx.x == 0) {
      if (!mbar_wait(never, 0, 20ull * 1000 * 1000, abort_flag)) {
        pair_record_error(a.err, abort_flag, rank, 4);
        aborted = true;
      }
    }
    for (int tile = pair; tile < total_tiles && !aborted; tile += num_pairs) {
      const int kblocks = KG ? (s_mts[tile / kg_per_group] + kGemmBK - 1) / kGemmBK
                             : tile < sh_tiles ? a.sh_J * a.sh_num_kb : a.num_kb;
      if (!mbar_wait(&acc_empty[acc], acc_ph ^ 1u, a.timeout_ns, abort_flag)) {
        pair_record_error(a.err, abort_flag, rank, 5);
        aborted = true;
        break;
      }
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * kGemmBN);
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!mbar_wait(&full[s], ph, a.timeout_ns, abort_flag)) {
          pair_record_error(a.err, abort_flag, rank, 6);
          aborted = true;
          break;
        }
        tc_fence_after_sync();
        // K-major: 16 K columns are 32 bytes along a row (+2 in 16-byte units); MN-major: 16 K rows of
        // 128 bytes (+128), the two 64-element MN chunks of a stage 8 KB apart
        const uint64_t ad = mn_a ? sw128_mnmajor_desc(smem_u32(sA + s * kStageA), kStageA / 2)
                                 : sw128_kmajor_desc(smem_u32(sA + s * kStageA));
        const uint64_t bd = mn_b ? sw128_mnmajor_desc(smem_u32(sB + s * kStageB), kStageB / 2)
                                 : sw128_kmajor_desc(smem_u32(sB + s * kStageB));
        const uint64_t astep = mn_a ? 128u : 2u, bstep = mn_b ? 128u : 2u;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16_ss_pair(d_tmem, ad + astep * kk, bd + bstep * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
        umma_commit_pair_multicast(&empty[s], 0x3);
        if (++s == kGemmStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (aborted) break;
      umma_commit_pair_multicast(&acc_full[acc], 0x3);
      if (++acc == 2) {
        acc = 0;
        acc_ph ^= 1u;
      }
    }
    umma_commit_pair_multicast(teardown, 0x1);
    mbar_wait_drain(teardown, 0, a.timeout_ns);
  } else if (warp >= 2) {
    // ------------------------------ epilogue ----------------------------------
    const int q = warp & 3;
    const int r = q * 32 + lane;
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int tile = pair; tile < total_tiles; tile += num_pairs) {
      const TileCoord c = KG ? TileCoord{} : decode_tile(tile, sh_tiles, s_mts, s_rows, G, a.n_tiles);
      bool ok = mbar_wait(&acc_full[acc], acc_ph, a.timeout_ns, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) pair_record_error(a.err, abort_flag, rank, 7);
        aborted = true;
        break;
      }
      tc_fence_after_sync();
      const uint32_t tb = tmem + static_cast<uint32_t>(acc * kGemmBN) + (static_cast<uint32_t>(q * 32) << 16);
      const size_t row = static_cast<size_t>(c.row0) + rank * kCtaRows + r;

      if (KG) {
        // fp32 weight gradient rows; a group without rows is all zeros (no MMA wrote the accumulator)
        const int g = tile / kg_per_group, local = tile - g * kg_per_group;
        const int mt = local / a.n_tiles, nt = local - mt * a.n_tiles;
        const int m = mt * kGemmBM + static_cast<int>(rank) * kCtaRows + r;
        const bool empty_group = s_mts[g] == 0;
        float* orow = nullptr;
        if (m < a.kg_M)
          orow = m < a.kg_split
                     ? a.kg_out + (static_cast<size_t>(g) * a.kg_split + m) * a.kg_ld
                     : a.kg_out2 + (static_cast<size_t>(g) * (a.kg_M - a.kg_split) + (m - a.kg_split)) * a.kg_ld;
#pragma unroll 1
        for (int cc = 0; cc < kGemmBN; cc += 16) {
          uint32_t vr[16];
          tmem_ld16(tb + cc, vr);
          tmem_ld_wait();
          const int col = nt * kGemmBN + cc;
          if (orow && col < a.n_limit) {
            float4* dst = reinterpret_cast<float4*>(orow + col);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = empty_group ? make_float4(0.f, 0.f, 0.f, 0.f)
                                   : make_float4(__uint_as_float(vr[4 * j]), __uint_as_float(vr[4 * j + 1]),
                                                 __uint_as_float(vr[4 * j + 2]), __uint_as_float(vr[4 * j + 3]));
          }
        }
      } else {
        const int n0 = c.n_tile * kGemmBN;
        const float sc = c.shared || !a.row_scale ? 1.f : a.row_scale[row];
        __nv_bfloat16* orow = (c.shared ? a.sh_out : a.out) + row * a.ld_out;
#pragma unroll 1
        for (int cc = 0; cc < kGemmBN; cc += 16) {
          uint32_t vr[16];
          tmem_ld16(tb + cc, vr);
          tmem_ld_wait();
          const int col = n0 + cc;
          if (col < a.n_limit) {
            uint32_t pk[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
              pk[j] = pack_bf16x2(sc * __uint_as_float(vr[2 * j]), sc * __uint_as_float(vr[2 * j + 1]));
            uint4* dst = reinterpret_cast<uint4*>(orow + col);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_lead + 8u * static_cast<uint32_t>(acc));
      if (++acc == 2) {
        acc = 0;
        acc_ph ^= 1u;
      }
    }
  }
  if (aborted || *abort_flag) {
    // a copy issued by this CTA may still be landing: give it time before the
    // pair leaves (copies take microseconds; this path only follows a timeout)
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200ull * 1000) {
    }
  }
  tc_fence_before_sync();
  cluster_sync();  // the even CTA's MMAs and both epilogues are done with TMEM and shared memory
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace fgs
