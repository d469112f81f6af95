// fp8_gemm.cuh -- the layer's expert FFNs with fine-grained FP8 operands.
//
// DeepSeek-V3 technical report, section 3.3 "FP8 Training": the GEMMs take
// FP8 inputs, each small group of values with its own power-of-two scale,
// and accumulate in high precision; Appendix B.2 "Discussion About Block-Wise
// Quantization": activations are grouped 1 x 128 along the channels in the
// forward pass, weights in 128 x 128 blocks.  The router stays in bf16/fp32.
//
// Three kernels replace the bf16 path's permutation and expert GEMMs:
//   permute_quant_kernel      the routing permutation of permute.cuh, copying
//                             each token row as E4M3 codes with one UE8M0
//                             scale per 128 columns, quantized once and
//                             written to the token's K expert rows and to the
//                             dense rows the shared experts read
//   fp8_gemm_kernel<true>     H = SiLU(u W_gate^T) * (u W_up^T), then H itself
//                             quantized 1 x 128 in the epilogue (the down
//                             projection's operand): codes and scales
//   fp8_gemm_kernel<false>    Y = g * (H W_down^T) (routed) and Ys (shared);
//                             the final sum is the bf16 path's combine_kernel
// The GEMMs are block-scaled tcgen05 MMAs (kind::mxf8f6f4, E4M3, UE8M0 scales
// read from TMEM), M = 128 rows, N = 256 (gate/up: 128 W_gate rows and the
// same 128 W_up rows; down: 256 output columns), 128 K per stage: one
// activation group and one weight block.
//
// Activation scales are kept in the hardware's scale-atom layout: for a
// matrix of R rows and C columns, atom (R / 128, C / 128) of 512 bytes holds
// the scales of its 128 rows for that 128-column group (fp8_util.cuh), so a
// stage copies its A scales with one 512-byte bulk copy.  Weight scales come
// as the quantizer writes them (one byte per 128 x 128 block); the producer
// warp spreads a block's byte over an atom in shared memory.
//
// One persistent CTA per SM, 320 threads, tiles in a static round-robin
// order (the shared experts' tiles first):
//   warp 0      producer: TMA boxes [128 rows, 128 B] of A and B (128-byte
//               swizzle), the A scale atom (bulk copy), the B scale atoms
//               (written by the warp), into a 4-stage ring
//   warp 1      allocates 512 TMEM columns: one 256-column accumulator and
//               two 12-column scale slots; one lane copies each stage's scales
//               into a slot (tcgen05.cp) and issues 4 block-scaled MMAs
//   warps 2-9   epilogue: two warps per 32-lane quadrant, each taking half
//               of the accumulator's columns for its rows; both drain the
//               accumulator to registers first and free it, so the next
//               tile's MMAs start while they compute
#pragma once

#include "fp8_util.cuh"
#include "permute.cuh"
#include "sm100.cuh"

namespace fgs {

constexpr int kF8Threads = 320;
constexpr int kF8Stages = 4;
constexpr int kF8BM = 128;  // rows of A per tile (MMA M)
constexpr int kF8BN = 256;  // MMA N
constexpr int kF8BK = 128;  // K per stage: one scale group
constexpr uint32_t kF8BoxA = kF8BM * kF8BK;            // 16 KB
constexpr uint32_t kF8BoxB = kF8BN * kF8BK;            // 32 KB: two 128-row boxes (gate/up) or one 256-row box
constexpr uint32_t kF8SfA = kSfAtomBytes;              // the A rows' scales of the stage's group
constexpr uint32_t kF8SfB = 2 * kSfAtomBytes;          // the B rows' scales: two atoms of 128 rows
constexpr uint32_t kF8Stage = 51200;                   // A + B + scales, padded to 1 KB
static_assert(kF8BoxA + kF8BoxB + kF8SfA + kF8SfB <= kF8Stage && kF8Stage % 1024 == 0, "stage layout");
constexpr uint32_t kF8TmemCols = 512;
constexpr uint32_t kF8SfCol = 256;                     // scale slot j at column 256 + 12 j: A 4, B 8 columns
constexpr uint32_t kF8BoxRowsW = 128;                  // W_gate / W_up boxes; W_down boxes are 256 rows
constexpr uint32_t kF8BoxRowsWd = 256;

__host__ __device__ constexpr size_t fp8_gemm_smem_bytes() {
  return 1024 + static_cast<size_t>(kF8Stages) * kF8Stage + 8 * (2 * kF8Stages + 2 + 2) + 16 +
         4 * (2 * 264) + 4 * 2 * 2 * 128 + 4 * 2 * 4 * 2;
}
static_assert(fp8_gemm_smem_bytes() <= 232448, "shared memory");

// ---------------------------------------------------------------------------
// The permutation with FP8 rows
// ---------------------------------------------------------------------------
struct PermuteQuantArgs {
  PermuteArgs p;            // the ranking of permute.cuh (p.gather unused)
  uint8_t* xq_perm;         // [P, d] codes of the expert-ordered rows
  uint8_t* xs_perm;         // scale atoms of xq_perm: [P / 128][d / 128][512]
  uint8_t* xq;              // [T_pad, d] codes of the rows of x (the shared experts' A), or null
  uint8_t* xs;              // scale atoms of xq
};

// Writes the 4-byte scale cell of row R of group g into an atom array of
// `groups` groups per 128-row block.
__device__ __forceinline__ void put_scale(uint8_t* atoms, size_t R, int g, int groups, uint32_t byte) {
  uint8_t* atom = atoms + ((R >> 7) * static_cast<size_t>(groups) + g) * kSfAtomBytes;
  *reinterpret_cast<uint32_t*>(atom + sf_atom_offset(static_cast<int>(R & 127))) = 0x01010101u * byte;
}

// grid (nblk, split), as permute_gather_kernel; d is a multiple of 128.
__global__ void __launch_bounds__(kPermThreads) permute_quant_kernel(PermuteQuantArgs q) {
  const PermuteArgs& a = q.p;
  __shared__ uint32_t masks[256 * 4];
  __shared__ int32_t base[256], roff[256], rstart[256];
  __shared__ int32_t dst[kPermBlockTokens * 8];
  const int tid = threadIdx.x;
  const int b = blockIdx.x, sp = blockIdx.y;
  const int t0 = b * kPermBlockTokens;
  const int ntok = min(kPermBlockTokens, a.T - t0);
  const int K = a.K;

  pdl_launch_dependents();
  pdl_wait();  // the router's outputs are complete and visible from here
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
  __syncthreads();
  // quantize each token row once: a warp per row, 256 columns (two groups)
  // per pass, lanes 0-15 holding the first group and lanes 16-31 the second
  const int warp = tid >> 5, lane = tid & 31, nwarps = kPermThreads / 32;
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
          const size_t R = static_cast<size_t>(dst[tl * K + k]);
          *reinterpret_cast<uint2*>(q.xq_perm + R * a.d + col) = codes;
          if ((lane & 15) == 0) put_scale(q.xs_perm, R, g, groups, sbyte);
        }
        if (q.xq) {
          *reinterpret_cast<uint2*>(q.xq + t * a.d + col) = codes;
          if ((lane & 15) == 0) put_scale(q.xs, t, g, groups, sbyte);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// The block-scaled GEMMs
// ---------------------------------------------------------------------------
struct Fp8GemmArgs {
  // routed experts (grouped rows; their tiles follow the shared ones)
  int num_groups;              // experts; 0: no routed tiles
  const int32_t* mtile_start;  // [G + 1] prefix sum of ceil(count / 128)
  const int32_t* row_start;    // [G + 1] first row of each expert
  int n_tiles;                 // gate/up: 128 H columns per tile; down: 256 output columns
  int num_kg;                  // 128-wide K groups of a routed tile (gate/up: d / 128; down: I / 128)
  const uint8_t* a_atoms;      // scale atoms of the routed A rows (xs_perm or hs_perm)
  int a_groups;                // K groups per row of the routed A (its atom array's width)
  const uint8_t* w_scale0;     // routed weight block scales: gate/up W_gate [G][I/128][d/128]; down W_down [G][d/128][I/128]
  const uint8_t* w_scale1;     // gate/up: W_up's; down: unused
  int w_rows128;               // 128-row blocks of one expert's weight matrix (gate/up: I/128; down: d/128)
  const float* row_scale;      // down: g of each row of Y
  // gate/up outputs: H codes and scale atoms; down outputs: Y (bf16)
  uint8_t* hq;
  uint8_t* hs_atoms;
  int h_groups, sh_h_groups;   // gate/up: 128-column groups per row of H (I / 128) and of Hs (K_s I_s / 128)
  __nv_bfloat16* y;
  int ld_out, n_limit;         // row stride and valid columns of the routed output
  // shared experts (dense rows; tiles first)
  int sh_rows;                 // tokens; 0: no shared tiles
  int sh_n_tiles;
  int sh_J;                    // down: shared experts summed in one accumulator (gate/up: 1)
  int sh_kg_per_j;             // K groups per shared expert (gate/up: d / 128; down: I_s / 128)
  int sh_k_per_j;              // down: A columns per shared expert (I_s)
  const uint8_t* sh_a_atoms;   // scale atoms of the shared A rows (xs or hss)
  int sh_a_groups;
  const uint8_t* sh_w_scale0;  // gate/up: W_gate,s [K_s][I_s/128][d/128]; down: W_down,s [K_s][d/128][I_s/128]
  const uint8_t* sh_w_scale1;  // gate/up: W_up,s
  int sh_w_rows128;            // 128-row blocks of one shared expert's matrix (gate/up: I_s/128; down: d/128)
  uint8_t* sh_hq;              // gate/up: Hs codes [T_pad, K_s I_s]
  uint8_t* sh_hs_atoms;
  __nv_bfloat16* sh_y;         // down: Ys
  int sh_ld_out, sh_n_limit;
  uint32_t* err;
  uint64_t timeout_ns;
  int debug_wait;              // test only: CTA 0 waits 20 ms on a barrier nothing arrives on
};

struct F8Tile {
  int shared, g, m_tile, n_tile, row0;
};

__device__ __forceinline__ F8Tile f8_decode(int tile, int sh_tiles, int sh_n_tiles, const int32_t* s_mts,
                                           const int32_t* s_rows, int G, int n_tiles) {
  F8Tile c;
  if (tile < sh_tiles) {
    c.shared = 1;
    c.g = 0;
    c.m_tile = tile / sh_n_tiles;
    c.n_tile = tile - c.m_tile * sh_n_tiles;
    c.row0 = c.m_tile * kF8BM;
    return c;
  }
  tile -= sh_tiles;
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
  c.row0 = s_rows[lo] + c.m_tile * kF8BM;
  return c;
}

__device__ __forceinline__ void f8_record_error(uint32_t* err, volatile int* abort, uint32_t site) {
  *abort = 1;
  atomicOr(err, kErrTimeout | (1u << (kErrSiteShift + site)));
}

__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// GU: tmA = X_perm codes, tmAs = x codes ([rows][d], 128-row boxes); tmB /
// tmB2 = W_gate / W_up codes [G][I][d] and tmBs / tmBs2 the shared ones
// [1][K_s I_s][d] (128-row boxes).  !GU: tmA = H codes [P][I], tmAs = Hs codes
// [T_pad][K_s I_s]; tmB = W_down codes [G][d][I], tmBs = [K_s][d][I_s]
// (256-row boxes); tmB2 / tmBs2 unused.
template <bool GU>
__global__ void __launch_bounds__(kF8Threads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmAs,
                    const __grid_constant__ CUtensorMap tmBs, const __grid_constant__ CUtensorMap tmBs2,
                    Fp8GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kF8Stages * kF8Stage);
  uint64_t* empty = full + kF8Stages;
  uint64_t* acc_full = empty + kF8Stages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* teardown = acc_empty + 1;
  uint64_t* never = teardown + 1;  // test only: a barrier nothing arrives on
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_mts = reinterpret_cast<int32_t*>(tmem_slot + 4);  // [264]
  int32_t* s_rows = s_mts + 264;
  // per tile parity (so that a warp one tile ahead never overwrites what its partner still reads):
  float* s_amax = reinterpret_cast<float*>(s_rows + 264);                  // [2][2][128] the halves' row maxima
  volatile int* s_ok = reinterpret_cast<volatile int*>(s_amax + 2 * 2 * 128);  // [2][4][2] each warp's wait result

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.num_groups;
  const int sh_tiles = a.sh_rows > 0 ? (a.sh_rows + kF8BM - 1) / kF8BM * a.sh_n_tiles : 0;
  if (tid == 0) {
    for (int s = 0; s < kF8Stages; ++s) {
      mbar_init(&full[s], 2);  // the producer's expect_tx arrive and its arrive after writing the B scales
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);  // one arrive per epilogue warp
    mbar_init(teardown, 1);
    mbar_init(never, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kF8TmemCols);
    tmem_relinquish();
  }
  pdl_wait();  // the permuted rows, their scales and the router's tables are complete from here
  pdl_launch_dependents();
  for (int i = tid; i <= G; i += kF8Threads) {
    s_mts[i] = G ? a.mtile_start[i] : 0;
    s_rows[i] = G ? a.row_start[i] : 0;
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int total_tiles = sh_tiles + s_mts[G] * a.n_tiles;

  if (warp == 0) {
    // ------------------------------ producer ----------------------------------
    int s = 0, issued = 0;
    uint32_t ph = 0;
    bool stop = false;
    if (lane == 0) {
      if (G) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (GU) tma_prefetch_desc(&tmB2);
      }
      if (sh_tiles) {
        tma_prefetch_desc(&tmAs);
        tma_prefetch_desc(&tmBs);
        if (GU) tma_prefetch_desc(&tmBs2);
      }
    }
    for (int tile = blockIdx.x; tile < total_tiles && !stop; tile += gridDim.x) {
      const F8Tile c = f8_decode(tile, sh_tiles, a.sh_n_tiles, s_mts, s_rows, G, a.n_tiles);
      const int J = c.shared ? a.sh_J : 1;
      const int kgs = c.shared ? a.sh_kg_per_j : a.num_kg;
      const int n0 = c.n_tile * (GU ? kF8BN / 2 : kF8BN);
      for (int j = 0; j < J && !stop; ++j) {
        // the B rows' block scales of every K group of this tile (and shared expert j), loaded once:
        // lane l holds groups l and l + 32 (at most 64 groups: d, I, I_s <= 8192); a stage takes
        // its byte by a shuffle instead of a global load on the producer's critical path
        uint32_t sc0[2] = {127u, 127u}, sc1[2] = {127u, 127u};
        {
          const uint8_t* s0 = c.shared ? a.sh_w_scale0 : a.w_scale0;
          const int rows128 = c.shared ? a.sh_w_rows128 : a.w_rows128;
          const int groups = c.shared ? a.sh_kg_per_j : a.num_kg;
          size_t base0, base1;
          if (GU) {
            // the shared experts' rows are K_s blocks of I_s side by side: block n0 / 128 of the whole
            const size_t blk = c.shared ? static_cast<size_t>(n0 >> 7) : static_cast<size_t>(c.g) * rows128 + (n0 >> 7);
            base0 = base1 = blk * groups;
          } else {
            const size_t mat = static_cast<size_t>(c.shared ? j : c.g) * rows128;
            const int r0 = n0 >> 7;
            base0 = (mat + r0) * groups;
            base1 = r0 + 1 < rows128 ? (mat + r0 + 1) * groups : base0;  // rows past d are zero: any scale
          }
          const uint8_t* s1 = GU ? (c.shared ? a.sh_w_scale1 : a.w_scale1) : s0;
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int kgl = lane + 32 * h2;
            if (kgl < kgs) {
              sc0[h2] = __ldg(s0 + base0 + kgl);
              sc1[h2] = __ldg(s1 + base1 + kgl);
            }
          }
        }
        for (int kg = 0; kg < kgs; ++kg) {
          bool ok = true;
          if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1u, a.timeout_ns, abort_flag);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) {
            if (lane == 0) f8_record_error(a.err, abort_flag, 3);
            stop = true;
            break;
          }
          uint8_t* st = smem + s * kF8Stage;
          uint8_t* sfa = st + kF8BoxA + kF8BoxB;
          uint8_t* sfb = sfa + kF8SfA;
          // A column (within its row): routed kg * 128; shared down j * I_s + kg * 128
          const int acol = (c.shared && !GU) ? j * a.sh_k_per_j + kg * kF8BK : kg * kF8BK;
          const int agroup = acol / kF8BK;
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[s], kF8BoxA + kF8BoxB + kF8SfA);
            tma_load_2d(st, c.shared ? &tmAs : &tmA, &full[s], acol, c.row0);
            if (GU) {
              tma_load_3d(st + kF8BoxA, c.shared ? &tmBs : &tmB, &full[s], kg * kF8BK, n0, c.g);
              tma_load_3d(st + kF8BoxA + kF8BoxB / 2, c.shared ? &tmBs2 : &tmB2, &full[s], kg * kF8BK, n0, c.g);
            } else {
              tma_load_3d(st + kF8BoxA, c.shared ? &tmBs : &tmB, &full[s], kg * kF8BK, n0, c.shared ? j : c.g);
            }
            const uint8_t* atoms = c.shared ? a.sh_a_atoms : a.a_atoms;
            const int agroups = c.shared ? a.sh_a_groups : a.a_groups;
            bulk_copy_g2s(sfa, atoms + (static_cast<size_t>(c.row0 >> 7) * agroups + agroup) * kSfAtomBytes, kF8SfA,
                          &full[s]);
          }
          // the B rows' scales: one byte per 128 x 128 weight block, spread over its atom
          const uint32_t b0 = __shfl_sync(0xffffffffu, kg < 32 ? sc0[0] : sc0[1], kg & 31);
          const uint32_t b1 = __shfl_sync(0xffffffffu, kg < 32 ? sc1[0] : sc1[1], kg & 31);
          const uint32_t w0 = 0x01010101u * b0, w1 = 0x01010101u * b1;
          reinterpret_cast<uint4*>(sfb)[lane] = make_uint4(w0, w0, w0, w0);
          reinterpret_cast<uint4*>(sfb + kSfAtomBytes)[lane] = make_uint4(w1, w1, w1, w1);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[s]);
          ++issued;
          if (++s == kF8Stages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
    if (lane == 0) {
      for (int st = 0; st < kF8Stages; ++st) {
        if (issued > st) {
          const int n = (issued - 1 - st) / kF8Stages + 1;
          mbar_wait_drain(&full[st], static_cast<uint32_t>((n - 1) & 1), a.timeout_ns);
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------ MMA issuer --------------------------------
    const uint32_t idesc = idesc_mxf8_e4m3(kF8BM, kF8BN);
    int s = 0, slot = 0;
    uint32_t ph = 0, acc_ph = 0;
    bool stop = false;
    if (a.debug_wait && blockIdx.x == 0 && !mbar_wait(never, 0, 20ull * 1000 * 1000, abort_flag)) {
      f8_record_error(a.err, abort_flag, 10);
      stop = true;
    }
    for (int tile = blockIdx.x; tile < total_tiles && !stop; tile += gridDim.x) {
      const int kgs = tile < sh_tiles ? a.sh_J * a.sh_kg_per_j : a.num_kg;
      if (!mbar_wait(acc_empty, acc_ph ^ 1u, a.timeout_ns, abort_flag)) {
        f8_record_error(a.err, abort_flag, 5);
        break;
      }
      acc_ph ^= 1u;
      tc_fence_after_sync();
      for (int kg = 0; kg < kgs; ++kg) {
        if (!mbar_wait(&full[s], ph, a.timeout_ns, abort_flag)) {
          f8_record_error(a.err, abort_flag, 6);
          stop = true;
          break;
        }
        tc_fence_after_sync();
        const uint32_t st = smem_u32(smem + s * kF8Stage);
        const uint32_t tsfa = tmem + kF8SfCol + 12u * slot, tsfb = tsfa + 4u;
        tmem_cp_sf(tsfa, sf_atom_desc(st + kF8BoxA + kF8BoxB));
        tmem_cp_sf(tsfb, sf_atom_desc(st + kF8BoxA + kF8BoxB + kF8SfA));
        tmem_cp_sf(tsfb + 4u, sf_atom_desc(st + kF8BoxA + kF8BoxB + kF8SfA + kSfAtomBytes));
        const uint64_t ad = sw128_kmajor_desc(st), bd = sw128_kmajor_desc(st + kF8BoxA);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_mxf8_ss(tmem, ad + 2 * kk, bd + 2 * kk, idesc, tsfa, tsfb, (kg | kk) != 0 ? 1u : 0u);
        umma_commit(&empty[s]);
        slot ^= 1;
        if (++s == kF8Stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (stop) break;
      umma_commit(acc_full);
    }
    umma_commit(teardown);
    mbar_wait_drain(teardown, 0, a.timeout_ns);
  } else if (warp >= 2) {
    // ------------------------------ epilogue ----------------------------------
    const int q = warp & 3;             // TMEM lanes 32 q .. + 31
    const int h = (warp - 2) >> 2;      // which half of the accumulator's columns
    const int r = q * 32 + lane;        // row of the tile
    const uint32_t bar_id = 1u + static_cast<uint32_t>(q);  // the quadrant's two warps
    uint32_t acc_ph = 0;
    int par = 0;  // tile parity: which copy of s_ok and s_amax this tile uses
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, par ^= 1) {
      const F8Tile c = f8_decode(tile, sh_tiles, a.sh_n_tiles, s_mts, s_rows, G, a.n_tiles);
      bool ok = mbar_wait(acc_full, acc_ph, a.timeout_ns, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      // both warps of the quadrant take the same decision at the same barrier
      volatile int* okp = s_ok + par * 8 + q * 2;
      if (lane == 0) okp[h] = ok ? 1 : 0;
      asm volatile("bar.sync %0, 64;" ::"r"(bar_id) : "memory");
      const bool both = okp[0] && okp[1];
      if (!both) {
        if (lane == 0 && !ok) f8_record_error(a.err, abort_flag, 7);
        break;
      }
      acc_ph ^= 1u;
      tc_fence_after_sync();
      const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16);
      const size_t row = static_cast<size_t>(c.row0) + r;
      if (GU) {
        // gate columns [64 h, 64 h + 64), up columns [128 + 64 h, ...): H columns n0 + 64 h ..
        // the raw accumulator into registers first and the accumulator freed, so that the next
        // tile's MMAs run while this tile's SwiGLU and quantization are computed
        uint32_t gr[64], ur[64];
#pragma unroll
        for (int cc = 0; cc < 64; cc += 16) {
          tmem_ld16(tb + 64 * h + cc, *reinterpret_cast<uint32_t(*)[16]>(gr + cc));
          tmem_ld16(tb + 128 + 64 * h + cc, *reinterpret_cast<uint32_t(*)[16]>(ur + cc));
        }
        tmem_ld_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);  // the accumulator is in registers
        float hv[64];
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const float g = __uint_as_float(gr[j]), u = __uint_as_float(ur[j]);
          hv[j] = g / (1.f + __expf(-g)) * u;
        }
        // the row's 1 x 128 group is this tile's 128 H columns: the two halves' maxima
        float m = 0.f;
#pragma unroll
        for (int j = 0; j < 64; ++j) m = fmaxf(m, fabsf(hv[j]));
        float* am = s_amax + par * 256;
        am[h * 128 + r] = m;
        asm volatile("bar.sync %0, 64;" ::"r"(bar_id) : "memory");
        m = fmaxf(am[r], am[128 + r]);
        const int e = scale_exponent(m);
        const float inv = pow2_neg(e);
        const int n0 = c.n_tile * (kF8BN / 2);
        const int n_limit = c.shared ? a.sh_n_limit : a.n_limit;
        const int ld = c.shared ? a.sh_ld_out : a.ld_out;
        uint8_t* orow = (c.shared ? a.sh_hq : a.hq) + row * ld + n0 + 64 * h;
        if (n0 + 64 * h < n_limit) {
#pragma unroll
          for (int j = 0; j < 64; j += 16) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 p0 = make_float2(hv[j + 4 * i] * inv, hv[j + 4 * i + 1] * inv);
              const float2 p1 = make_float2(hv[j + 4 * i + 2] * inv, hv[j + 4 * i + 3] * inv);
              const uint32_t c0 = uint32_t(__nv_cvt_float2_to_fp8x2(p0, __NV_SATFINITE, __NV_E4M3)) & 0xFFFFu;
              const uint32_t c1 = uint32_t(__nv_cvt_float2_to_fp8x2(p1, __NV_SATFINITE, __NV_E4M3)) & 0xFFFFu;
              w[i] = c0 | (c1 << 16);
            }
            *reinterpret_cast<uint4*>(orow + j) = make_uint4(w[0], w[1], w[2], w[3]);
          }
          if (h == 0) {
            const int groups = c.shared ? a.sh_h_groups : a.h_groups;
            put_scale(c.shared ? a.sh_hs_atoms : a.hs_atoms, row, n0 / kF8BK, groups,
                      static_cast<uint32_t>(e + 127));
          }
        }
      } else {
        // columns [128 h, 128 h + 128) of the tile: output columns n0 + 128 h ..
        const int n0 = c.n_tile * kF8BN + 128 * h;
        const int n_limit = c.shared ? a.sh_n_limit : a.n_limit;
        const int ld = c.shared ? a.sh_ld_out : a.ld_out;
        // the raw accumulator into registers and the accumulator freed before the gate's load
        uint32_t v[128];
#pragma unroll
        for (int cc = 0; cc < 128; cc += 16)
          tmem_ld16(tb + 128 * h + cc, *reinterpret_cast<uint32_t(*)[16]>(v + cc));
        tmem_ld_wait();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        const float sc = c.shared ? 1.f : a.row_scale[row];
        uint32_t pk[64];
#pragma unroll
        for (int j = 0; j < 64; ++j)
          pk[j] = pack_bf16x2(sc * __uint_as_float(v[2 * j]), sc * __uint_as_float(v[2 * j + 1]));
        if (n0 < n_limit) {
          __nv_bfloat16* orow = (c.shared ? a.sh_y : a.y) + row * ld + n0;
#pragma unroll
          for (int j = 0; j < 64; j += 4)
            *reinterpret_cast<uint4*>(orow + 2 * j) = make_uint4(pk[j], pk[j + 1], pk[j + 2], pk[j + 3]);
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kF8TmemCols);
  }
}

}  // namespace fgs
