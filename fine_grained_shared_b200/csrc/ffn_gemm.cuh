// ffn_gemm.cuh -- steps 4 and 5 of the layer: the expert FFNs as grouped
// GEMMs on the 5th-generation tensor cores, with the SwiGLU, the gate scale
// and the final sum fused into the epilogues.
//
// FFN_i(u) = W_down,i (SiLU(W_gate,i u) * (W_up,i u)) for every routed expert
// i (the fine-grained experts of DeepSeekMoE, arXiv 2401.06066, Abstract and
// blog section "Fine-Grained Expert Segmentation (Section 3.1)") and for the
// always-active shared experts (blog section "Shared Expert Isolation
// (Section 3.2)").
//
// One persistent kernel template, one CTA per SM, 192 threads:
//   warp 0      TMA producer: A tile [128 rows, 64] and B tile [256 rows, 64]
//               per k-block into a 4-stage ring (128-byte swizzle)
//   warp 1      allocates 512 TMEM columns; one lane issues tcgen05.mma
//               (M = 128, N = 256, K = 16) into one of two 256-column fp32
//               accumulators, so the epilogue of tile i overlaps the MMAs of
//               tile i + 1
//   warps 2-5   epilogue; warp w reads TMEM lanes 32*(w%4) .. +31 (one
//               output row per thread)
// Tiles are (group, m-tile, n-tile).  A "group" is one routed expert (its
// rows are read from device-side offsets written by the router, so the host
// never synchronises) or the single dense group of the shared experts.
//
// Epilogues:
//   SWIGLU   B = [W_gate rows n0..n0+127 ; W_up rows n0..n0+127]:
//            H[row, n0 + c] = SiLU(acc[c]) * acc[128 + c]   (bf16)
//   SCALE    Y[row, n0 + c] = g[row] * acc[c]               (bf16)
//   COMBINE  out[t, n0 + c] = x[t] + acc[c] + sum_k Y[slot[t, k], n0 + c]
//            (the shared experts' down projection carries the final,
//            deterministic, k-ordered sum of the layer)
#pragma once

#include "sm100.cuh"

namespace fgs {

constexpr int kGemmThreads = 192;
constexpr int kGemmStages = 4;
constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;  // MMA N (SWIGLU: 128 gate + 128 up columns)
constexpr int kGemmBK = 64;
constexpr uint32_t kStageA = kGemmBM * kGemmBK * 2;   // 16 KB
constexpr uint32_t kStageB = kGemmBN * kGemmBK * 2;   // 32 KB
constexpr uint32_t kTmemCols = 512;

enum EpiKind { EPI_SWIGLU = 0, EPI_SCALE = 1, EPI_COMBINE = 2 };

struct GemmArgs {
  // schedule
  int grouped;                 // 1: groups from mtile_start/row_start; 0: one dense group
  int num_groups;              // groups when grouped
  const int32_t* mtile_start;  // [num_groups + 1]
  const int32_t* row_start;    // [num_groups + 1]
  int dense_rows;              // rows of the dense group
  int n_tiles;                 // output tiles along N per group
  int num_kb;                  // 64-wide k-blocks per sub-expert
  int J;                       // sub-experts summed into one accumulator
  int k_per_j;                 // A columns per sub-expert
  // epilogue
  int n_limit;                 // valid output columns
  __nv_bfloat16* out;
  int ld_out;
  const float* row_scale;      // SCALE
  const __nv_bfloat16* x;      // COMBINE
  const __nv_bfloat16* y;      // COMBINE
  const int32_t* slot_of;      // COMBINE [T, K]
  int K, T, d;
  int add_residual, add_routed;
  // errors
  uint32_t* err;
  uint64_t timeout_ns;
  int debug_wait;              // CTA 0 waits on a barrier nothing arrives on
};

__host__ __device__ constexpr size_t gemm_smem_bytes() {
  return 1024 + static_cast<size_t>(kGemmStages) * (kStageA + kStageB) + 8 * (2 * kGemmStages + 4 + 2) + 16 +
         4 * 2 * 264;
}

__device__ __forceinline__ void gemm_record_error(uint32_t* err, volatile int* abort, uint32_t site) {
  *abort = 1;
  atomicOr(err, kErrTimeout | (1u << (kErrSiteShift + site)));
}

struct TileCoord {
  int g, m_tile, n_tile, row0;
};

__device__ __forceinline__ TileCoord decode_tile(int tile, const int32_t* s_mts, const int32_t* s_rows, int G,
                                                 int n_tiles) {
  // largest g with s_mts[g] * n_tiles <= tile (empty groups share a start)
  int lo = 0, hi = G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_mts[mid] * n_tiles <= tile) lo = mid;
    else hi = mid;
  }
  TileCoord c;
  c.g = lo;
  const int local = tile - s_mts[lo] * n_tiles;
  c.m_tile = local / n_tiles;
  c.n_tile = local - c.m_tile * n_tiles;
  c.row0 = s_rows[lo] + c.m_tile * kGemmBM;
  return c;
}

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    ffn_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1, GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kGemmStages * kStageA;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kGemmStages * kStageB);
  uint64_t* empty = full + kGemmStages;
  uint64_t* acc_full = empty + kGemmStages;   // [2]
  uint64_t* acc_empty = acc_full + 2;         // [2]
  uint64_t* never = acc_empty + 2;
  uint64_t* teardown = never + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(teardown + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_mts = reinterpret_cast<int32_t*>(tmem_slot + 4);  // [264]
  int32_t* s_rows = s_mts + 264;                                // [264]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  int G;
  if (a.grouped) {
    G = a.num_groups;
    for (int i = tid; i <= G; i += kGemmThreads) {
      s_mts[i] = a.mtile_start[i];
      s_rows[i] = a.row_start[i];
    }
  } else {
    G = 1;
    if (tid == 0) {
      s_mts[0] = 0;
      s_mts[1] = (a.dense_rows + kGemmBM - 1) / kGemmBM;
      s_rows[0] = 0;
      s_rows[1] = s_mts[1] * kGemmBM;
    }
  }
  if (tid == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4 * 32);
    }
    mbar_init(never, 1);
    mbar_init(teardown, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int total_tiles = s_mts[G] * a.n_tiles;

  if (warp == 0 && lane == 0) {
    // ------------------------------ TMA producer ------------------------------
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (EPI == EPI_SWIGLU) tma_prefetch_desc(&tmB1);
    int s = 0, issued = 0;
    uint32_t ph = 0;
    bool stop = false;
    for (int tile = blockIdx.x; tile < total_tiles && !stop; tile += gridDim.x) {
      const TileCoord c = decode_tile(tile, s_mts, s_rows, G, a.n_tiles);
      for (int j = 0; j < a.J && !stop; ++j) {
        for (int kb = 0; kb < a.num_kb; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, a.timeout_ns, abort_flag)) {
            gemm_record_error(a.err, abort_flag, 3);
            stop = true;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kStageA + kStageB);
          const int kc = kb * kGemmBK;
          tma_load_2d(sA + s * kStageA, &tmA, &full[s], j * a.k_per_j + kc, c.row0);
          if (EPI == EPI_SWIGLU) {
            const int n0 = c.n_tile * (kGemmBN / 2);
            tma_load_3d(sB + s * kStageB, &tmB0, &full[s], kc, n0, c.g);
            tma_load_3d(sB + s * kStageB + kStageB / 2, &tmB1, &full[s], kc, n0, c.g);
          } else {
            tma_load_3d(sB + s * kStageB, &tmB0, &full[s], kc, c.n_tile * kGemmBN, c.g * a.J + j);
          }
          ++issued;
          if (++s == kGemmStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
    for (int st = 0; st < kGemmStages; ++st) {
      if (issued > st) {
        const int n = (issued - 1 - st) / kGemmStages + 1;
        mbar_wait(&full[st], static_cast<uint32_t>((n - 1) & 1), a.timeout_ns, nullptr);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------ MMA issuer --------------------------------
    const uint32_t idesc = idesc_bf16_f32(kGemmBM, kGemmBN);
    int s = 0, acc = 0;
    uint32_t ph = 0, acc_ph = 0;
    bool stop = false;
    if (a.debug_wait && blockIdx.x == 0) {
      if (!mbar_wait(never, 0, 20ull * 1000 * 1000, abort_flag)) {
        gemm_record_error(a.err, abort_flag, 4);
        stop = true;
      }
    }
    for (int tile = blockIdx.x; tile < total_tiles && !stop; tile += gridDim.x) {
      if (!mbar_wait(&acc_empty[acc], acc_ph ^ 1u, a.timeout_ns, abort_flag)) {
        gemm_record_error(a.err, abort_flag, 5);
        break;
      }
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * kGemmBN);
      bool first = true;
      for (int j = 0; j < a.J && !stop; ++j) {
        for (int kb = 0; kb < a.num_kb; ++kb) {
          if (!mbar_wait(&full[s], ph, a.timeout_ns, abort_flag)) {
            gemm_record_error(a.err, abort_flag, 6);
            stop = true;
            break;
          }
          tc_fence_after_sync();
          const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + s * kStageA));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + s * kStageB));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            umma_bf16_ss(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, first ? 0u : 1u);
            first = false;
          }
          umma_commit(&empty[s]);
          if (++s == kGemmStages) {
            s = 0;
            ph ^= 1u;
          }
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
    mbar_wait(teardown, 0, a.timeout_ns, nullptr);
  } else if (warp >= 2) {
    // ------------------------------ epilogue ----------------------------------
    const int q = warp & 3;
    const int r = q * 32 + lane;
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const TileCoord c = decode_tile(tile, s_mts, s_rows, G, a.n_tiles);
      bool ok = mbar_wait(&acc_full[acc], acc_ph, a.timeout_ns, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0) gemm_record_error(a.err, abort_flag, 7);
        break;
      }
      tc_fence_after_sync();
      const uint32_t tb = tmem + static_cast<uint32_t>(acc * kGemmBN) + (static_cast<uint32_t>(q * 32) << 16);
      const size_t row = static_cast<size_t>(c.row0) + r;

      if (EPI == EPI_SWIGLU) {
        const int n0 = c.n_tile * (kGemmBN / 2);
        __nv_bfloat16* orow = a.out + row * a.ld_out;
#pragma unroll 1
        for (int cc = 0; cc < kGemmBN / 2; cc += 16) {
          uint32_t gr[16], ur[16];
          tmem_ld16(tb + cc, gr);
          tmem_ld16(tb + kGemmBN / 2 + cc, ur);
          tmem_ld_wait();
          const int col = n0 + cc;
          if (col < a.n_limit) {
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
      } else if (EPI == EPI_SCALE) {
        const int n0 = c.n_tile * kGemmBN;
        const float sc = a.row_scale[row];
        __nv_bfloat16* orow = a.out + row * a.ld_out;
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
      } else {  // EPI_COMBINE: rows are tokens
        const int n0 = c.n_tile * kGemmBN;
        const int t = static_cast<int>(row);
        const bool tok_ok = t < a.T;
        int slots[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          slots[k] = (tok_ok && a.add_routed && k < a.K) ? a.slot_of[static_cast<size_t>(t) * a.K + k] : -1;
#pragma unroll 1
        for (int cc = 0; cc < kGemmBN; cc += 16) {
          uint32_t vr[16];
          tmem_ld16(tb + cc, vr);
          tmem_ld_wait();
          const int col = n0 + cc;
          if (tok_ok && col < a.n_limit) {
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = 0.f;
            if (a.add_residual) {
              const uint4* xr = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * a.d + col);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint4 w4 = __ldg(xr + h);
                const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  v[8 * h + 2 * j] += bf16lo(w[j]);
                  v[8 * h + 2 * j + 1] += bf16hi(w[j]);
                }
              }
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] += __uint_as_float(vr[j]);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              if (slots[k] >= 0) {
                const uint4* yr = reinterpret_cast<const uint4*>(a.y + static_cast<size_t>(slots[k]) * a.d + col);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const uint4 w4 = __ldcg(yr + h);
                  const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                  for (int j = 0; j < 4; ++j) {
                    v[8 * h + 2 * j] += bf16lo(w[j]);
                    v[8 * h + 2 * j + 1] += bf16hi(w[j]);
                  }
                }
              }
            }
            uint32_t pk[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) pk[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
            uint4* dst = reinterpret_cast<uint4*>(a.out + static_cast<size_t>(t) * a.ld_out + col);
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
    tc_fence_before_sync();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace fgs
