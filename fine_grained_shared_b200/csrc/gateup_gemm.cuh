// gateup_gemm.cuh -- step 4 of the layer: the expert FFNs' first half,
// H = SiLU(u W_gate^T) * (u W_up^T), as a grouped GEMM on the 5th-generation
// tensor cores with the SwiGLU fused into the epilogue.
//
// FFN_i(u) = W_down,i (SiLU(W_gate,i u) * (W_up,i u)) for every routed expert
// i (the fine-grained experts of DeepSeekMoE, arXiv 2401.06066, Abstract and
// blog section "Fine-Grained Expert Segmentation (Section 3.1)") and for the
// always-active shared experts (blog section "Shared Expert Isolation
// (Section 3.2)").
//
// One persistent kernel, one CTA per SM, 192 threads:
//   warp 0      TMA producer.  Per 64-column k-block it stages the A tile
//               [128 rows, 64] (routed experts: rows of the expert-ordered
//               copy of x; shared experts: rows of x) and B = [W_gate rows
//               n0..n0+127 ; W_up rows n0..n0+127] in a 4-stage ring
//               (128-byte swizzle).
//   warp 1      allocates 512 TMEM columns; one lane issues tcgen05.mma
//               (M = 128, N = 256: gate and up side by side, K = 16) into one
//               of two 256-column fp32 accumulators, so the epilogue of tile
//               i overlaps the MMAs of tile i + 1
//   warps 2-5   epilogue; warp w reads TMEM lanes 32*(w%4) .. +31 (one H row
//               per thread) and stores bf16 SiLU(gate) * up
// One launch covers both kinds of expert.  Its tiles are (part, group,
// 128-row m-tile, 128-column n-tile): first the shared experts' tiles over
// the rows of x (one dense group whose H columns are the shared experts'
// intermediate columns side by side), then the routed experts' tiles, whose
// groups' m-tile starts come from the router on the device, so the host never
// synchronises.  The shared experts' tiles go round-robin over the CTAs and
// need neither the router nor the permutation, so under programmatic
// dependent launch they run while those kernels finish; the producer then
// waits for them and takes routed tiles dynamically: the SMs of each of the
// B200's two dies take tiles from their own half of the routed range (so the
// two dies' L2 halves do not both fetch every expert's weights) and steal
// from the other half when theirs runs out.  The producer passes each tile id
// to the MMA and epilogue warps through a 4-entry shared-memory queue.
#pragma once

#include "sm100.cuh"

namespace fgs {

constexpr int kGuThreads = 192;
constexpr int kGuStages = 4;
constexpr int kGuBM = 128;
constexpr int kGuBN = 256;  // MMA N: 128 gate + 128 up columns
constexpr int kGuBK = 64;
constexpr uint32_t kGuStageA = kGuBM * kGuBK * 2;  // 16 KB
constexpr uint32_t kGuStageB = kGuBN * kGuBK * 2;  // 32 KB
constexpr uint32_t kGuTmemCols = 512;
// TMA box heights the host must encode
constexpr uint32_t kGuBoxRowsA = kGuBM;      // tiled x (shared experts)
constexpr uint32_t kGuBoxRowsB = kGuBN / 2;  // W_gate and W_up

struct GateUpArgs {
  // routed experts (grouped rows of X_perm; their tiles follow the shared ones)
  int num_groups;              // experts; 0: no routed tiles
  const int32_t* mtile_start;  // [G + 1] prefix sum of ceil(count / 128)
  const int32_t* row_start;    // [G + 1] first row of each expert in X_perm and H
  int n_tiles;                 // 128-column H tiles per expert
  int n_limit;                 // valid H columns
  __nv_bfloat16* out;          // H
  int ld_out;
  // shared experts (the dense rows of x; their tiles come first)
  int sh_rows;                 // tokens; 0: no shared tiles
  int sh_n_tiles;              // 128-column Hs tiles
  int sh_n_limit;              // valid Hs columns (shared experts x their intermediate size)
  __nv_bfloat16* sh_out;       // Hs
  int sh_ld_out;
  // both parts
  int num_kb;                  // 64-wide k-blocks over d
  int* tile_ctr;               // [2] per-die counters of the routed tiles, zeroed by the permutation
  int die_split;               // SMs with smid below this are on the first die
  uint32_t* err;
  uint64_t timeout_ns;
  int debug_wait;              // CTA 0 waits on a barrier nothing arrives on
  // the backward's recompute (gateup_gemm_kernel<true>): the incoming gradient of each H element and
  // what the epilogue writes instead of H
  const __nv_bfloat16* dm;     // routed: dL/dm per row of X_perm before the gate scale, [rows, n_limit]
  int ld_dm;
  const __nv_bfloat16* sh_dm;  // shared: dL/dm per token, [T, sh_n_limit]
  int sh_ld_dm;
  const float* row_gate;       // routed: the gate of each row
  float* dg_part;              // routed: [rows, n_tiles] per 128-column tile, sum of dm * m over its columns
  int sh_I;                    // shared: columns of one shared expert (I_s)
  // for the weight gradients (nullptr: not written): m row by row, and zeros in every output row
  // (m, da, db) that holds no (token, slot) pair, since the weight-gradient GEMMs sum over rows
  const int32_t* counts;       // routed: [G] rows of each expert (the rest of its segment is padding)
  __nv_bfloat16* m_out;        // routed: [rows, n_limit]
  __nv_bfloat16* sh_m_out;     // shared: [T_pad, sh_n_limit]
};

constexpr int kGuQueue = 4;  // tile-id queue entries

__host__ __device__ constexpr size_t gateup_smem_bytes() {
  return 1024 + static_cast<size_t>(kGuStages) * (kGuStageA + kGuStageB) +
         8 * (2 * kGuStages + 4 + 2 + 2 * kGuQueue) + 16 + 4 * (3 * 264 + kGuQueue);
}

__device__ __forceinline__ void gu_record_error(uint32_t* err, volatile int* abort, uint32_t site) {
  *abort = 1;
  atomicOr(err, kErrTimeout | (1u << (kErrSiteShift + site)));
}

struct GuTile {
  int shared;  // 1: a shared-expert tile over the rows of x
  int g, m_tile, n_tile, row0;
};

// tiles [0, sh_tiles) are the shared experts' (m-tile major); the rest are
// the routed experts', expert by expert
__device__ __forceinline__ GuTile gu_decode(int tile, int sh_tiles, int sh_n_tiles, const int32_t* s_mts,
                                           const int32_t* s_rows, int G, int n_tiles) {
  GuTile c;
  if (tile < sh_tiles) {
    c.shared = 1;
    c.g = 0;
    c.m_tile = tile / sh_n_tiles;
    c.n_tile = tile - c.m_tile * sh_n_tiles;
    c.row0 = c.m_tile * kGuBM;
    return c;
  }
  tile -= sh_tiles;
  int lo = 0, hi = G;  // largest g with s_mts[g] * n_tiles <= tile
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
  c.row0 = s_rows[lo] + c.m_tile * kGuBM;
  return c;
}

// tmA: X_perm with a 128-row box; tmG, tmU: W_gate, W_up as [experts][I][d]
// with a 128-row box.  tmAs: x with a 128-row box; tmGs, tmUs: the shared
// experts' W_gate, W_up as [1][K_s * I_s][d].  Maps of an absent part are
// never read.
//
// BWD = false: the forward, H = SiLU(a) * b from the accumulators a = A W_gate^T
// and b = A W_up^T.  BWD = true: the backward's recompute of a and b, whose
// epilogue takes the gradient dm of m = SiLU(a) * b (routed rows: before the
// gate scale g) and writes, per element, da = g dm b SiLU'(a) and
// db = g dm SiLU(a), SiLU'(a) = sigma(a) (1 + a (1 - sigma(a))): routed rows
// [da | db] as [rows, 2 I]; shared rows expert by expert, [da_j | db_j] for
// j < K_s; and, per routed row and 128-column tile, the partial sum of dm * m
// that makes the gate's gradient dg = dh . y (y = W_down m).
template <bool BWD>
__global__ void __launch_bounds__(kGuThreads, 1)
    gateup_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmG,
                       const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmAs,
                       const __grid_constant__ CUtensorMap tmGs, const __grid_constant__ CUtensorMap tmUs,
                       GateUpArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kGuStages * kGuStageA;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kGuStages * kGuStageB);
  uint64_t* empty = full + kGuStages;
  uint64_t* acc_full = empty + kGuStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint64_t* never = acc_empty + 2;
  uint64_t* teardown = never + 1;
  uint64_t* tq_full = teardown + 1;        // [kGuQueue] a tile id is in the slot
  uint64_t* tq_empty = tq_full + kGuQueue;  // [kGuQueue] MMA + 4 epilogue warps have read it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tq_empty + kGuQueue);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_mts = reinterpret_cast<int32_t*>(tmem_slot + 4);  // [264]
  int32_t* s_rows = s_mts + 264;                                // [264]
  volatile int32_t* s_tq = s_rows + 264;                        // [kGuQueue]
  int32_t* s_cnt = const_cast<int32_t*>(s_tq) + kGuQueue;       // [264] the backward's row counts

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  const int G = a.num_groups;
  const int sh_tiles = a.sh_rows > 0 ? (a.sh_rows + kGuBM - 1) / kGuBM * a.sh_n_tiles : 0;
  if (tid == 0) {
    for (int s = 0; s < kGuStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4 * 32);
    }
    mbar_init(never, 1);
    mbar_init(teardown, 1);
    for (int i = 0; i < kGuQueue; ++i) {
      mbar_init(&tq_full[i], 1);
      mbar_init(&tq_empty[i], 1 + 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kGuTmemCols);
    tmem_relinquish();
  }
  pdl_launch_dependents();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    // lane 0 issues every copy and hands each tile id to the MMA and epilogue
    // warps; the whole warp loads the routed experts' tables
    int s = 0, issued = 0, q = 0;
    uint32_t ph = 0, qph = 0;
    bool stop = false;
    auto publish = [&](int tile) {  // tile -1: no more tiles
      if (!mbar_wait(&tq_empty[q], qph ^ 1u, a.timeout_ns, abort_flag)) {
        gu_record_error(a.err, abort_flag, 8);
        stop = true;
        return;
      }
      s_tq[q] = tile;
      mbar_arrive(&tq_full[q]);
      if (++q == kGuQueue) {
        q = 0;
        qph ^= 1u;
      }
    };
    auto load_tile = [&](int tile) {
      const GuTile c = gu_decode(tile, sh_tiles, a.sh_n_tiles, s_mts, s_rows, G, a.n_tiles);
      const int n0 = c.n_tile * (kGuBN / 2);
      const CUtensorMap* mA = c.shared ? &tmAs : &tmA;
      const CUtensorMap* mG = c.shared ? &tmGs : &tmG;
      const CUtensorMap* mU = c.shared ? &tmUs : &tmU;
      for (int kb = 0; kb < a.num_kb; ++kb) {
        if (!mbar_wait(&empty[s], ph ^ 1u, a.timeout_ns, abort_flag)) {
          gu_record_error(a.err, abort_flag, 3);
          stop = true;
          return;
        }
        mbar_arrive_expect_tx(&full[s], kGuStageA + kGuStageB);
        const int kc = kb * kGuBK;
        tma_load_2d(sA + s * kGuStageA, mA, &full[s], kc, c.row0);
        tma_load_3d(sB + s * kGuStageB, mG, &full[s], kc, n0, c.g);
        tma_load_3d(sB + s * kGuStageB + kGuStageB / 2, mU, &full[s], kc, n0, c.g);
        ++issued;
        if (++s == kGuStages) {
          s = 0;
          ph ^= 1u;
        }
      }
    };
    if (lane == 0) {
      if (G) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmG);
        tma_prefetch_desc(&tmU);
      }
      if (sh_tiles) {
        tma_prefetch_desc(&tmAs);
        tma_prefetch_desc(&tmGs);
        tma_prefetch_desc(&tmUs);
      }
      // the shared experts' tiles read only x and the shared weights, so they
      // run while the router and the permutation may still be running
      for (int tile = blockIdx.x; tile < sh_tiles && !stop; tile += gridDim.x) {
        publish(tile);
        if (!stop) load_tile(tile);
      }
    }
    // the routed experts' tiles need the router's tables, the permuted rows and
    // the tile counters the permutation zeroed
    pdl_wait();
    for (int i = lane; i <= G; i += 32) {
      s_mts[i] = G ? a.mtile_start[i] : 0;
      s_rows[i] = G ? a.row_start[i] : 0;
      if (BWD) s_cnt[i] = (i < G && a.counts) ? a.counts[i] : 0;
    }
    __syncwarp();
    if (lane == 0) {
      // each die owns half of the routed tiles and helps the other at the end
      const int routed = s_mts[G] * a.n_tiles;
      const int half = routed / 2;
      const int die = static_cast<int>(sm_id()) >= a.die_split ? 1 : 0;
      const int own_lo = sh_tiles + (die ? half : 0), own_hi = sh_tiles + (die ? routed : half);
      const int oth_lo = sh_tiles + (die ? 0 : half), oth_hi = sh_tiles + (die ? half : routed);
      while (!stop) {
        int tile = -1;
        const int t = own_lo + atomicAdd(&a.tile_ctr[die], 1);
        if (t < own_hi) {
          tile = t;
        } else {  // this die's half is done: help the other die
          const int u = oth_lo + atomicAdd(&a.tile_ctr[die ^ 1], 1);
          if (u < oth_hi) tile = u;
        }
        publish(tile);
        if (stop || tile < 0) break;
        load_tile(tile);
      }
      for (int st = 0; st < kGuStages; ++st) {
        if (issued > st) {
          const int n = (issued - 1 - st) / kGuStages + 1;
          mbar_wait_drain(&full[st], static_cast<uint32_t>((n - 1) & 1), a.timeout_ns);
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------ MMA issuer --------------------------------
    const uint32_t idesc = idesc_bf16_f32(kGuBM, kGuBN);
    int s = 0, acc = 0;
    uint32_t ph = 0, acc_ph = 0;
    bool stop = false;
    if (a.debug_wait && blockIdx.x == 0) {
      if (!mbar_wait(never, 0, 20ull * 1000 * 1000, abort_flag)) {
        gu_record_error(a.err, abort_flag, 4);
        stop = true;
      }
    }
    int q = 0;
    uint32_t qph = 0;
    while (!stop) {
      if (!mbar_wait(&tq_full[q], qph, a.timeout_ns, abort_flag)) {
        gu_record_error(a.err, abort_flag, 9);
        break;
      }
      const int tile = s_tq[q];
      mbar_arrive(&tq_empty[q]);
      if (++q == kGuQueue) {
        q = 0;
        qph ^= 1u;
      }
      if (tile < 0) break;
      if (!mbar_wait(&acc_empty[acc], acc_ph ^ 1u, a.timeout_ns, abort_flag)) {
        gu_record_error(a.err, abort_flag, 5);
        break;
      }
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * kGuBN);
      for (int kb = 0; kb < a.num_kb; ++kb) {
        if (!mbar_wait(&full[s], ph, a.timeout_ns, abort_flag)) {
          gu_record_error(a.err, abort_flag, 6);
          stop = true;
          break;
        }
        tc_fence_after_sync();
        const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + s * kGuStageA));
        const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + s * kGuStageB));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16_ss(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
        umma_commit(&empty[s]);
        if (++s == kGuStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (stop) break;
      umma_commit(&acc_full[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_ph ^= 1u;
      }
    }
    umma_commit(teardown);
    mbar_wait_drain(teardown, 0, a.timeout_ns);
  } else if (warp >= 2) {
    // ------------------------------ epilogue ----------------------------------
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int r = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_ph = 0;
    int q = 0;
    uint32_t qph = 0;
    while (true) {
      bool okq = mbar_wait(&tq_full[q], qph, a.timeout_ns, abort_flag);
      okq = __all_sync(0xffffffffu, okq);
      if (!okq) {
        if (lane == 0) gu_record_error(a.err, abort_flag, 10);
        break;
      }
      const int tile = s_tq[q];
      __syncwarp();
      if (lane == 0) mbar_arrive(&tq_empty[q]);
      if (++q == kGuQueue) {
        q = 0;
        qph ^= 1u;
      }
      if (tile < 0) break;
      const GuTile c = gu_decode(tile, sh_tiles, a.sh_n_tiles, s_mts, s_rows, G, a.n_tiles);
      bool ok = mbar_wait(&acc_full[acc], acc_ph, a.timeout_ns, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) gu_record_error(a.err, abort_flag, 7);
        break;
      }
      tc_fence_after_sync();
      const uint32_t tb = tmem + static_cast<uint32_t>(acc * kGuBN) + (static_cast<uint32_t>(quarter * 32) << 16);
      const size_t row = static_cast<size_t>(c.row0) + r;
      const int n0 = c.n_tile * (kGuBN / 2);
      const int n_limit = c.shared ? a.sh_n_limit : a.n_limit;
      __nv_bfloat16* orow = c.shared ? a.sh_out + row * a.sh_ld_out : a.out + row * a.ld_out;
      if constexpr (BWD) {
        const float gsc = c.shared ? 1.f : a.row_gate[row];
        const __nv_bfloat16* dmrow = c.shared ? a.sh_dm + row * a.sh_ld_dm : a.dm + row * a.ld_dm;
        // a row that holds no (token, slot) pair (expert padding, or past the tokens) stores zeros
        // in m, da and db, since the weight gradients' sums over rows would otherwise take it in
        const bool valid = c.shared ? static_cast<int>(row) < a.sh_rows
                                    : static_cast<int>(row) - s_rows[c.g] < s_cnt[c.g];
        __nv_bfloat16* mrow = c.shared ? (a.sh_m_out ? a.sh_m_out + row * a.sh_n_limit : nullptr)
                                       : (a.m_out ? a.m_out + row * a.n_limit : nullptr);
        float dg = 0.f;
#pragma unroll 1
        for (int cc = 0; cc < kGuBN / 2; cc += 16) {
          uint32_t gr[16], ur[16];
          tmem_ld16(tb + cc, gr);
          tmem_ld16(tb + kGuBN / 2 + cc, ur);
          tmem_ld_wait();
          const int col = n0 + cc;
          if (col < n_limit) {
            const uint4* src = reinterpret_cast<const uint4*>(dmrow + col);
            const uint4 d0 = src[0], d1 = src[1];
            const uint32_t dw[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
            uint32_t pa[8], pb[8], pm[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              float da2[2], db2[2], m2[2];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const float av = __uint_as_float(gr[2 * j + h]), bv = __uint_as_float(ur[2 * j + h]);
                const float dmr = h ? bf16hi(dw[j]) : bf16lo(dw[j]);
                const float sg = 1.f / (1.f + __expf(-av));
                const float silu = av * sg;
                m2[h] = silu * bv;
                dg = fmaf(dmr, m2[h], dg);
                const float dmv = gsc * dmr;
                db2[h] = dmv * silu;
                da2[h] = dmv * bv * sg * (1.f + av * (1.f - sg));
              }
              pa[j] = pack_bf16x2(da2[0], da2[1]);
              pb[j] = pack_bf16x2(db2[0], db2[1]);
              pm[j] = valid ? pack_bf16x2(m2[0], m2[1]) : 0u;
            }
            if (mrow) {
              uint4* q = reinterpret_cast<uint4*>(mrow + col);
              q[0] = make_uint4(pm[0], pm[1], pm[2], pm[3]);
              q[1] = make_uint4(pm[4], pm[5], pm[6], pm[7]);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                pa[j] = valid ? pa[j] : 0u;
                pb[j] = valid ? pb[j] : 0u;
              }
            }
            __nv_bfloat16* pda;
            __nv_bfloat16* pdb;
            if (c.shared) {  // shared expert j's [da_j | db_j]
              const int j = col / a.sh_I, i = col - j * a.sh_I;
              pda = orow + static_cast<size_t>(j) * 2 * a.sh_I + i;
              pdb = pda + a.sh_I;
            } else {
              pda = orow + col;
              pdb = orow + a.n_limit + col;
            }
            reinterpret_cast<uint4*>(pda)[0] = make_uint4(pa[0], pa[1], pa[2], pa[3]);
            reinterpret_cast<uint4*>(pda)[1] = make_uint4(pa[4], pa[5], pa[6], pa[7]);
            reinterpret_cast<uint4*>(pdb)[0] = make_uint4(pb[0], pb[1], pb[2], pb[3]);
            reinterpret_cast<uint4*>(pdb)[1] = make_uint4(pb[4], pb[5], pb[6], pb[7]);
          }
        }
        if (!c.shared) a.dg_part[row * a.n_tiles + c.n_tile] = dg;
      } else {
#pragma unroll 1
      for (int cc = 0; cc < kGuBN / 2; cc += 16) {
        uint32_t gr[16], ur[16];
        tmem_ld16(tb + cc, gr);
        tmem_ld16(tb + kGuBN / 2 + cc, ur);
        tmem_ld_wait();
        const int col = n0 + cc;
        if (col < n_limit) {
          uint32_t pk[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float g0 = __uint_as_float(gr[2 * j]), g1 = __uint_as_float(gr[2 * j + 1]);
            const float u0 = __uint_as_float(ur[2 * j]), u1 = __uint_as_float(ur[2 * j + 1]);
            const float h0 = g0 / (1.f + __expf(-g0)) * u0;
            const float h1 = g1 / (1.f + __expf(-g1)) * u1;
            pk[j] = pack_bf16x2(h0, h1);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + col);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      }
      tc_fence_before_sync();
      mbar_arrive(&acc_empty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_ph ^= 1u;
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kGuTmemCols);
  }
}

}  // namespace fgs
