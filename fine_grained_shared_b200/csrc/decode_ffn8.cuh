// decode_ffn8.cuh -- the decode FFN of the FP8 layer: steps 4-5 for a decode
// batch on E4M3 codes with UE8M0 scales (1 x 128 groups of activation rows,
// 128 x 128 blocks of weights; DeepSeek-V3 technical report summary, section
// 3.3 "FP8 Training"), in one persistent launch.
//
// The schedule is decode_ffn_kernel's (decode_ffn.cuh): whole tiles [128
// weight rows x <= 32 tokens] numbered shared gate/up, routed gate/up, shared
// down, routed down, taken in turn from a global counter; a down tile waits on
// its token block's readiness counter.  The shared experts' tiles do not run
// ahead of the grid dependency wait here: their x codes come from the
// quantizing permutation.  What changes with FP8 operands:
//   - a k-block is one 128-column scale group (128 bytes of codes per row);
//     a stage holds one gate/up group (the W_gate and W_up boxes [128, 128 B],
//     the token box [32, 128 B]) or two down groups, and the scale atoms of
//     its groups;
//   - the MMA is tcgen05.mma.kind::mxf8f6f4.block_scale (M = 128 weight rows,
//     N = 32 tokens, K = 32); its scales are copied into TMEM per stage
//     (tcgen05.cp) from 512-byte atoms that the producer warp writes: the
//     weights' from the block's one scale byte, the tokens' with each lane's
//     scale cell (read through L2 from the activation atoms, 16 groups per
//     round trip) at rows 0-31, column 0 of the atom, so the MMA reads them
//     at the slot's own column (a tile's 32 rows sit in one column of their
//     128-row atom; reading them there would offset the scale address by one
//     column, and only even offsets are known to be valid);
//   - the gate/up epilogue quantizes H: a tile's 128 weight rows are the 128
//     columns of one 1 x 128 group of every token, so the group maximum is a
//     maximum over the four epilogue warps.  Each warp reduces its 32 rows
//     (redux.sync) and merges them into a shared-memory cell per token with a
//     64-bit atomic max tagged by the tile's sequence number (no reset between
//     tiles), then waits (bounded) until all four warps have arrived; no named
//     barrier joins warps that may have given up.  The codes (E4M3 of
//     h 2^-e, round to nearest even, saturating) go to H's rows and each
//     token's scale byte into the atoms the down tiles read.
// TMEM: seven accumulator buffers of 64 columns (448) and four 16-column
// scale slots, one per ring stage.
#pragma once

#include "decode_ffn.cuh"
#include "fp8_gemm.cuh"

namespace fgs {

constexpr uint32_t kF8dBoxW = 128 * 128;  // 16 KB: 128 weight rows x 128 codes
constexpr uint32_t kF8dBoxX = 32 * 128;   // 4 KB: 32 token rows x 128 codes
// stage layout: gate/up: W_gate 0, W_up 16 KB, tokens 32 KB, scale atoms W_gate / W_up / tokens at
// 36 KB + 0 / 512 / 1024; down (groups h = 0, 1): W_down h 20 KB, H h 20 KB + 16 KB, scale atoms at
// 40 KB + 1 KB h (weights) and + 512 (tokens)
constexpr uint32_t kF8dStage = 43008;
constexpr uint32_t kF8dSfOff = 36864;     // gate/up scale atoms
constexpr uint32_t kF8dDnSfOff = 40960;   // down scale atoms
static_assert(kF8dSfOff + 3 * kSfAtomBytes <= kF8dStage && kF8dDnSfOff + 4 * kSfAtomBytes <= kF8dStage, "stage");
constexpr int kF8dStages = 4;
constexpr int kF8dAccBufs = 7;            // 448 accumulator columns
constexpr uint32_t kF8dSfCol = 448;       // stage s's scales at columns 448 + 16 s
constexpr uint32_t kF8dTmemCols = 512;

__host__ __device__ constexpr size_t ffn8_smem_bytes() {
  return 1024 + static_cast<size_t>(kF8dStages) * kF8dStage +
         8 * (2 * kF8dStages + 2 * kF8dAccBufs + 2 * kFfnItems + 2) + 16 + sizeof(FfnItem) * kFfnItems +
         4 * (3 * (kFfnMaxExperts + 8)) + 8 * 64 + 16;
}
static_assert(ffn8_smem_bytes() <= 232448, "shared memory");
static_assert(2 * ffn8_smem_bytes() > 233472, "two CTAs would fit on one SM");

struct Ffn8Args {
  FfnArgs f;  // the schedule, the outputs Y / Ys (H / Hs unused: codes below), counters
  // activation codes' scale atoms (512 bytes per 128 rows and 128 columns)
  const uint8_t* x_atoms;      // X_perm codes' atoms: [rows / 128][d / 128]
  const uint8_t* xs_atoms;     // x codes' atoms (shared experts' gate/up): [T_pad / 128][d / 128]
  uint8_t* hq;                 // [rows, I] codes of H
  uint8_t* h_atoms;            // [rows / 128][I / 128]
  uint8_t* hsq;                // [T_pad, K_s I_s] codes of Hs
  uint8_t* hs_atoms;           // [T_pad / 128][K_s I_s / 128]
  // weight block scales (one byte per 128 x 128 block)
  const uint8_t* s_gate;       // [G][I / 128][d / 128]
  const uint8_t* s_up;
  const uint8_t* s_down;       // [G][d / 128][I / 128]
  const uint8_t* sh_s_gate;    // [K_s I_s / 128][d / 128]
  const uint8_t* sh_s_up;
  const uint8_t* sh_s_down;    // [K_s][d / 128][I_s / 128]
};

// Maps: tmWg / tmWu the routed experts' W_gate / W_up codes as [G][I][d]
// (128-row boxes), tmX X_perm codes, tmWsg / tmWsu the shared experts' as
// [1][K_s I_s][d], tmXs x codes; tmWd W_down codes as [G][d][I] (128-row
// boxes), tmH H codes, tmWsd W_down,s codes as [K_s][d][I_s], tmHs Hs codes.
// Token boxes 32 rows; all boxes 128 bytes wide.
__global__ void __launch_bounds__(kFfnThreads, 1)
    decode_ffn8_kernel(const __grid_constant__ CUtensorMap tmWg, const __grid_constant__ CUtensorMap tmWu,
                       const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWsg,
                       const __grid_constant__ CUtensorMap tmWsu, const __grid_constant__ CUtensorMap tmXs,
                       const __grid_constant__ CUtensorMap tmWd, const __grid_constant__ CUtensorMap tmH,
                       const __grid_constant__ CUtensorMap tmWsd, const __grid_constant__ CUtensorMap tmHs,
                       Ffn8Args a8) {
  const FfnArgs& a = a8.f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kF8dStages * kF8dStage);
  uint64_t* empty = full + kF8dStages;
  uint64_t* acc_full = empty + kF8dStages;        // [kF8dAccBufs]
  uint64_t* acc_empty = acc_full + kF8dAccBufs;   // [kF8dAccBufs]
  uint64_t* item_full = acc_empty + kF8dAccBufs;  // [kFfnItems]
  uint64_t* item_empty = item_full + kFfnItems;   // [kFfnItems]
  uint64_t* teardown = item_empty + kFfnItems;
  uint64_t* never = teardown + 1;  // test only: a barrier nothing arrives on
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  FfnItem* items = reinterpret_cast<FfnItem*>(tmem_slot + 4);
  int32_t* s_tbs = reinterpret_cast<int32_t*>(items + kFfnItems);
  int32_t* s_rows = s_tbs + kFfnMaxExperts + 8;
  int32_t* s_cnt = s_rows + kFfnMaxExperts + 8;
  unsigned long long* s_amax = reinterpret_cast<unsigned long long*>(
      (reinterpret_cast<uintptr_t>(s_cnt + kFfnMaxExperts + 8) + 7) & ~uintptr_t(7));  // [2][32]
  uint32_t* s_arrive = reinterpret_cast<uint32_t*>(s_amax + 64);                          // [2]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kF8dStages; ++s) {
      mbar_init(&full[s], 2);  // the producer's expect_tx arrive and its arrive after writing the weight scales
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < kF8dAccBufs; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    for (int i = 0; i < kFfnItems; ++i) {
      mbar_init(&item_full[i], 1);
      mbar_init(&item_empty[i], 5);
    }
    mbar_init(teardown, 1);
    mbar_init(never, 1);
    *abort_flag = 0;
    for (int i = 0; i < 64; ++i) s_amax[i] = 0ull;
    s_arrive[0] = s_arrive[1] = 0u;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kF8dTmemCols);
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
  const int d_groups = a.kb_gu;  // d / 128

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
    if (lane == 0 && sb) {
      tma_prefetch_desc(&tmWsg);
      tma_prefetch_desc(&tmWsu);
      tma_prefetch_desc(&tmXs);
    }
    // unlike the bf16 decode FFN's, the shared experts' gate/up tiles read what the previous kernel
    // writes (the codes and scales of x), so no tile starts before the grid dependency wait
    pdl_wait();
    auto routed = [&](long long t, int n_wb, FfnItem& f) {
      int lo = 0, hi = a.G;
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
      // the tile's scales go out before the item is published and the readiness wait, in one round trip
      // the tile's weight block scales, loaded once: lane l holds groups l and l + 32 (at most 64)
      uint32_t sc0[2] = {127u, 127u}, sc1[2] = {127u, 127u};
      {
        const int wrow_blk = f.wb;  // the tile's 128 weight rows are one row block
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int gl = lane + 32 * h2;
          if (gl < f.nkb) {
            if (f.kind == 0) {
              const size_t base = static_cast<size_t>(wrow_blk) * d_groups + gl;
              sc0[h2] = __ldg(a8.sh_s_gate + base);
              sc1[h2] = __ldg(a8.sh_s_up + base);
            } else if (f.kind == 1) {
              const size_t base = (static_cast<size_t>(f.g) * a.n_wb_gu + wrow_blk) * d_groups + gl;
              sc0[h2] = __ldg(a8.s_gate + base);
              sc1[h2] = __ldg(a8.s_up + base);
            } else if (f.kind == 2) {
              const int j = gl / a.sh_kb_per_j, kg = gl - j * a.sh_kb_per_j;
              sc0[h2] = __ldg(a8.sh_s_down + (static_cast<size_t>(j) * a.sh_n_wb_dn + wrow_blk) * a.sh_kb_per_j + kg);
            } else {
              sc0[h2] = __ldg(a8.s_down + (static_cast<size_t>(f.g) * a.n_wb_dn + wrow_blk) * a.kb_dn + gl);
            }
          }
        }
      }
      // the token rows' scales: lane n's cell (row row0 + n) in group k of the operand's atom array
      // [rows / 128][groups] is 4 bytes at 512 k from `cell0`
      const uint8_t* tok_atoms = f.kind == 0 ? a8.xs_atoms : f.kind == 1 ? a8.x_atoms : f.kind == 2 ? a8.hs_atoms
                                                                                                  : a8.h_atoms;
      const int tok_groups = f.kind < 2 ? d_groups : f.kind == 2 ? a.sh_cols / 128 : a.I / 128;
      const uint8_t* cell0 = tok_atoms + static_cast<size_t>(f.row0 >> 7) * tok_groups * kSfAtomBytes +
                             sf_atom_offset((f.row0 & 127) + lane);
      uint32_t cells[16];
      int cells_k0 = -16;
      auto load_cells = [&](int k0) {  // the cells of groups k0 .. k0 + 15, one round trip
        cells_k0 = k0;
#pragma unroll
        for (int i = 0; i < 16; ++i)
          cells[i] = k0 + i < f.nkb
                         ? __ldcg(reinterpret_cast<const unsigned int*>(cell0 + static_cast<size_t>(k0 + i) *
                                                                                    kSfAtomBytes))
                         : 0u;
      };
      // the activation rows' scales are complete (the grid dependency wait); H's only after its readiness
      if (f.kind >= 0 && f.kind < 2) load_cells(0);
      if (lane == 0) {
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
        if (!stop && (f.kind == 2 || f.kind == 3)) {
          // the down tile's rows of H and their scales: wait for every gate/up tile of its token block
          const uint32_t target = 4u * static_cast<uint32_t>(f.kind == 2 ? a.sh_n_wb_gu : a.n_wb_gu);
          if (!ffn_wait_ready(ready + f.ready, target, a.err, abort_flag, a.timeout_ns)) {
            ffn_record_error(a.err, abort_flag, 2);
            stop = true;
          }
          fence_proxy_async_global();
        }
      }
      stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
      if (stop) break;
      __syncwarp();  // lane 0's acquire of the readiness counter orders the other lanes' loads of H's scales too
      if (f.kind >= 2) load_cells(0);
      // stream the tile's groups: one per gate/up stage, two per down stage
      const int per = f.kind >= 2 ? 2 : 1;
      const int wrow = f.wb * kFfnWB;
      for (int kb = 0; kb < f.nkb; kb += per) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1u, a.timeout_ns, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) {
          if (lane == 0) ffn_record_error(a.err, abort_flag, 3);
          stop = true;
          break;
        }
        uint8_t* st = smem + s * kF8dStage;
        const int n = f.kind >= 2 ? min(2, f.nkb - kb) : 1;
        if (lane == 0) {
          if (f.kind < 2) {
            const int kc = kb * kF8BK;
            mbar_arrive_expect_tx(&full[s], 2 * kF8dBoxW + kF8dBoxX);
            tma_load_3d_hint(st, f.kind == 0 ? &tmWsg : &tmWg, &full[s], kc, wrow, f.g, pol_w);
            tma_load_3d_hint(st + kF8dBoxW, f.kind == 0 ? &tmWsu : &tmWu, &full[s], kc, wrow, f.g, pol_w);
            tma_load_2d(st + 2 * kF8dBoxW, f.kind == 0 ? &tmXs : &tmX, &full[s], kc, f.row0);
          } else {
            mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(n) * (kF8dBoxW + kF8dBoxX));
            for (int h = 0; h < n; ++h) {
              uint8_t* sh = st + h * (kF8dBoxW + kF8dBoxX);
              const int k = kb + h;
              if (f.kind == 2) {
                const int j = k / a.sh_kb_per_j, kc = (k - j * a.sh_kb_per_j) * kF8BK;
                tma_load_3d_hint(sh, &tmWsd, &full[s], kc, wrow, j, pol_w);
                tma_load_2d(sh + kF8dBoxW, &tmHs, &full[s], j * a.sh_k_per_j + kc, f.row0);
              } else {
                const int kc = k * kF8BK;
                tma_load_3d_hint(sh, &tmWd, &full[s], kc, wrow, f.g, pol_w);
                tma_load_2d(sh + kF8dBoxW, &tmH, &full[s], kc, f.row0);
              }
            }
          }
        }
        // the weights' scales: the block's byte spread over its atom (each lane 16 of the 512 bytes);
        // the tokens' scales: lane n's cell at row n, column 0 of the tokens' atom
        for (int h = 0; h < n; ++h) {
          const int k = kb + h;
          if (k >= cells_k0 + 16) load_cells(k & ~15);  // the next 16 groups' cells
          const uint32_t cell = cells[k - cells_k0];
          const uint32_t b0 = __shfl_sync(0xffffffffu, k < 32 ? sc0[0] : sc0[1], k & 31);
          const uint32_t w0 = 0x01010101u * b0;
          if (f.kind < 2) {
            const uint32_t b1 = __shfl_sync(0xffffffffu, k < 32 ? sc1[0] : sc1[1], k & 31);
            const uint32_t w1 = 0x01010101u * b1;
            reinterpret_cast<uint4*>(st + kF8dSfOff)[lane] = make_uint4(w0, w0, w0, w0);
            reinterpret_cast<uint4*>(st + kF8dSfOff + kSfAtomBytes)[lane] = make_uint4(w1, w1, w1, w1);
            *reinterpret_cast<uint32_t*>(st + kF8dSfOff + 2 * kSfAtomBytes + 16 * lane) = cell;
          } else {
            reinterpret_cast<uint4*>(st + kF8dDnSfOff + h * 2 * kSfAtomBytes)[lane] = make_uint4(w0, w0, w0, w0);
            *reinterpret_cast<uint32_t*>(st + kF8dDnSfOff + h * 2 * kSfAtomBytes + kSfAtomBytes + 16 * lane) = cell;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[s]);
        ++issued;
        if (++s == kF8dStages) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (lane == 0) {
      for (int st = 0; st < kF8dStages; ++st) {
        if (issued > st) {
          const int n = (issued - 1 - st) / kF8dStages + 1;
          mbar_wait_drain(&full[st], static_cast<uint32_t>((n - 1) & 1), a.timeout_ns);
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------ MMA issuer --------------------------------
    const uint32_t idesc = idesc_mxf8_e4m3(kFfnWB, kFfnTB);
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
        const uint32_t st = smem_u32(smem + s * kF8dStage);
        const uint32_t slot = tmem + kF8dSfCol + 16u * static_cast<uint32_t>(s);
        if (f.kind < 2) {
          tmem_cp_sf(slot, sf_atom_desc(st + kF8dSfOff));                      // W_gate
          tmem_cp_sf(slot + 4u, sf_atom_desc(st + kF8dSfOff + kSfAtomBytes));  // W_up
          tmem_cp_sf(slot + 8u, sf_atom_desc(st + kF8dSfOff + 2 * kSfAtomBytes));  // tokens
          const uint64_t xd = sw128_kmajor_desc(st + 2 * kF8dBoxW);
#pragma unroll
          for (int acc = 0; acc < 2; ++acc) {
            const uint64_t wd = sw128_kmajor_desc(st + acc * kF8dBoxW);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_mxf8_ss(d0 + acc * kFfnTB, wd + 2 * kk, xd + 2 * kk, idesc, slot + 4u * acc, slot + 8u,
                           (kb > 0 || kk > 0) ? 1u : 0u);
          }
        } else {
          const int n = min(2, f.nkb - kb);
          for (int h = 0; h < n; ++h) {
            const uint32_t sh = st + h * (kF8dBoxW + kF8dBoxX);
            const uint32_t sf = st + kF8dDnSfOff + h * 2 * kSfAtomBytes;
            tmem_cp_sf(slot + 8u * h, sf_atom_desc(sf));                       // W_down
            tmem_cp_sf(slot + 8u * h + 4u, sf_atom_desc(sf + kSfAtomBytes));   // H rows
            const uint64_t wd = sw128_kmajor_desc(sh), xd = sw128_kmajor_desc(sh + kF8dBoxW);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_mxf8_ss(d0, wd + 2 * kk, xd + 2 * kk, idesc, slot + 8u * h, slot + 8u * h + 4u,
                           (kb + h > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);
        if (++s == kF8dStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      umma_commit(&acc_full[buf]);
      if (++buf == kF8dAccBufs) {
        buf = 0;
        buf_ph ^= 1u;
      }
    }
    umma_commit(teardown);
    mbar_wait_drain(teardown, 0, a.timeout_ns);
  } else if (warp >= 2) {
    // ------------------------------ epilogue ----------------------------------
    const int q = warp & 3;
    const int r = q * 32 + lane;
    int buf = 0, it = 0;
    uint32_t buf_ph = 0, it_ph = 0;
    uint32_t gu_seq = 0;  // gate/up tiles seen: the tag of the shared group maxima
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
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      if (++buf == kF8dAccBufs) {
        buf = 0;
        buf_ph ^= 1u;
      }
      const int col = f.wb * kFfnWB + r;
      const bool shared = f.kind == 0 || f.kind == 2;
      if (gu) {
        // h = SiLU(g) u, then the 1 x 128 group maximum of every token over the four warps
#pragma unroll
        for (int j = 0; j < 32; ++j) v0[j] = __fdividef(v0[j], 1.f + __expf(-v0[j])) * v1[j];
        const uint32_t par = gu_seq & 1u;
        const unsigned long long tag = static_cast<unsigned long long>(gu_seq + 1) << 32;
        uint32_t mine = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(v0[j])));
          if (lane == j) mine = m;
        }
        atomicMax(&s_amax[par * 32 + lane], tag | mine);
        __threadfence_block();
        __syncwarp();
        if (lane == 0) atomicAdd(&s_arrive[par], 1u);
        // every warp's maxima are in once 4 (uses of this slot) arrivals are counted
        const uint32_t target = 4u * ((gu_seq >> 1) + 1u);
        bool arrived = true;
        if (lane == 0) {
          const uint64_t t0 = globaltimer_ns();
          while (*reinterpret_cast<volatile uint32_t*>(&s_arrive[par]) < target) {
            if (*abort_flag || globaltimer_ns() - t0 > a.timeout_ns) {
              arrived = false;
              break;
            }
            __nanosleep(32);
          }
        }
        arrived = __shfl_sync(0xffffffffu, arrived ? 1 : 0, 0) != 0;
        ++gu_seq;
        if (!arrived) {
          if (lane == 0) ffn_record_error(a.err, abort_flag, 9);
          break;
        }
        __threadfence_block();
        const uint32_t amax_lane = static_cast<uint32_t>(*reinterpret_cast<volatile unsigned long long*>(
            &s_amax[par * 32 + lane]));  // token `lane`'s group maximum
        const int n_limit = shared ? a.sh_cols : a.I;
        if (col < n_limit) {
          uint8_t* op = (shared ? a8.hsq : a8.hq) + static_cast<size_t>(f.row0) * n_limit + col;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int e = scale_exponent(__uint_as_float(__shfl_sync(0xffffffffu, amax_lane, j)));
            if (j < f.nvalid) {
              const float2 p = make_float2(v0[j] * pow2_neg(e), 0.f);
              *op = static_cast<uint8_t>(uint32_t(__nv_cvt_float2_to_fp8x2(p, __NV_SATFINITE, __NV_E4M3)) & 0xFFu);
              if (r == j)  // one thread per token writes its scale byte
                put_scale(shared ? a8.hs_atoms : a8.h_atoms, static_cast<size_t>(f.row0) + j, f.wb, n_limit / 128,
                          static_cast<uint32_t>(e + 127));
            }
            op += n_limit;
          }
        }
        // this warp's rows of the tile are in H: count them for the down tiles' TMA and bulk loads
        fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(ready + f.ready, 1u);
      } else {
        if (col < a.d) {
          __nv_bfloat16* op = (shared ? a.ys : a.y) + static_cast<size_t>(f.row0) * a.d + col;
          const float* rs = shared ? nullptr : a.row_scale + f.row0;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (j < f.nvalid) *op = __float2bfloat16_rn(shared ? v0[j] : rs[j] * v0[j]);
            op += a.d;
          }
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kF8dTmemCols);
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
