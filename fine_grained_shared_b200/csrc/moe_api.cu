// moe_api.cu -- the C ABI declared in include/fgs_moe.h: argument checks,
// workspace, TMA descriptors and the launch sequence of one layer forward.
//
// Launch sequence, all on the caller's stream:
//   router_topk (logits, top-K, histogram, scan)  idx, gate, offsets
//   permute_gather                                X_perm, slot_of, g
//   gate/up GEMM + SwiGLU, shared and routed      Hs = SwiGLU(x), H = SwiGLU(X_perm)
//   down GEMM, shared and routed (+ gate scale)   Ys = Hs W_down,s^T, Y = g * (H W_down^T)
//   combine                                       out = x + Ys + sum_k Y (k ascending)
// Each GEMM launch covers the shared experts' tiles and the routed experts'
// tiles in one persistent kernel, so the shared experts fill the SMs that a
// small batch's routed tiles leave idle and the two never wait on each
// other's tail.  Batches of up to 512 tokens launch every kernel with
// programmatic dependent launch, so each kernel's prologue overlaps the tail
// of the one before.  Nothing is copied back to the host.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/fgs_moe.h"
#include "backward.cuh"
#include "decode_ffn.cuh"
#include "decode_ffn8.cuh"
#include "down_gemm.cuh"
#include "ep.cuh"
#include "fp8_gemm.cuh"
#include "gateup_gemm.cuh"
#include "permute.cuh"
#include "router_topk.cuh"

using namespace fgs;

static_assert(kGemmBM == kExpertRowAlign, "GEMM pair tiles must not straddle two experts");
static_assert(kFfnBoxRowsW == kGuBoxRowsB && kFfnBoxRowsW == kBoxRowsB,
              "the decode FFN shares the weight maps of the prefill GEMMs");

// Batches of at most this many tokens run the expert FFNs on the
// weight-streaming decode kernel (decode_ffn.cuh); larger ones on the
// 128-row-tile GEMMs.
#ifndef FGS_DECODE_MAX_T
#define FGS_DECODE_MAX_T 64
#endif


namespace {

constexpr int kMaxRouted = 256;
constexpr int kMaxK = 8;
constexpr int64_t kMaxTokens = int64_t(1) << 20;
constexpr uint64_t kTimeoutNs = 2000ull * 1000 * 1000;  // 2 s: no legitimate wait comes close
constexpr int64_t kDecodeMaxT = FGS_DECODE_MAX_T;
// the host-buffer forward pipelines batches of at least 2 x kHostChunkRows tokens in up to kHostChunks chunks
constexpr int kHostChunks = 5;
constexpr int64_t kHostChunkRows = 2048;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool load_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// bf16 tensor [d2][rows][cols] (d2 = 1 for a matrix), box [1][box_rows][64],
// 128-byte swizzle, zero fill outside the tensor.
bool encode_bf16(CUtensorMap* m, const void* base, uint64_t d2, uint64_t rows, uint64_t cols, uint32_t box_rows,
                 int rank) {
  cuuint64_t dims[3] = {cols, rows, d2};
  cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// uint8 tensor [d2][rows][cols] (E4M3 codes), box [1][box_rows][128], 128-byte swizzle.
bool encode_u8(CUtensorMap* m, const void* base, uint64_t d2, uint64_t rows, uint64_t cols, uint32_t box_rows,
               int rank) {
  cuuint64_t dims[3] = {cols, rows, d2};
  cuuint64_t strides[2] = {cols, rows * cols};
  cuuint32_t box[3] = {128, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct MapCache {
  const void* ptr = nullptr;
  int64_t rows = -1;
  CUtensorMap map;
};

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
inline int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

struct Layout {
  // byte offsets into the workspace
  size_t err, done, tile_ctr, tok_done, small_logits, idx, gate, slot, src, bc, counts, offsets, row_start, mtile,
      mtile128, gate_perm, x_perm, h, y, hs, ys, xdev, outdev, ffn_ctr, xq_perm, xs_perm, xq, xs, hq, hs_perm, hsq,
      hss, ep_base, ep_counts, ep_row_start, ep_mtile, ep_mtile128, total;
  int64_t P, Pa, Tpad, nblk;
};

// Token blocks a decode batch can have: 32-token blocks of the shared
// experts' rows, and of each routed expert's rows (at most one partial block
// per expert that received a token).  Each has a readiness counter in the
// decode FFN, so a batch runs there only if they fit.
int64_t decode_token_blocks(int64_t T, int64_t K, int64_t N) {
  return (T + kFfnTB - 1) / kFfnTB + std::min<int64_t>(N, T * K) + (T * K + kFfnTB - 1) / kFfnTB;
}

Layout make_layout(const moe_config& c) {
  Layout L{};
  const int64_t Tm = c.max_tokens, Km = c.max_k, N = c.n_routed;
  L.nblk = ceil_div(Tm, 128);
  // sum over experts of ceil(count / 256) * 256 <= T*K + 255*N; an expert-parallel rank holds N / G
  // experts and may receive every rank's T*K rows
  const int64_t G = c.ep_ranks > 1 ? c.ep_ranks : 1;
  L.P = G * Tm * Km + (N / G) * (kExpertRowAlign - 1);
  L.Tpad = int64_t(ceil_div(Tm, kGemmBM)) * kGemmBM;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  L.err = take(16);
  L.done = take(16);
  L.tile_ctr = take(16);
  L.tok_done = take(kSmallRouterMaxT * 4);  // zeroed with the header block at creation
  L.small_logits = take(size_t(kSmallRouterMaxT) * N * 4);
  L.idx = take(Tm * Km * 4);
  L.gate = take(Tm * Km * 4);
  L.slot = take(Tm * Km * 4);
  L.src = take(Tm * Km * 4);
  L.bc = take(L.nblk * N * 4);
  L.counts = take(N * 4);
  L.offsets = take((N + 1) * 4);
  // expert parallelism: this rank's destination rows per expert, its own experts' tables
  L.ep_base = take(N * 4);
  L.ep_counts = take((N + 1) * 4);
  L.ep_row_start = take((N + 1) * 4);
  L.ep_mtile = take((N + 1) * 4);
  L.ep_mtile128 = take((N + 1) * 4);
  L.row_start = take((N + 1) * 4);
  L.mtile = take((N + 1) * 4);
  L.mtile128 = take((N + 1) * 4);
  L.gate_perm = take(L.P * 4);
  L.x_perm = take(L.P * c.d_model * 2);
  L.h = take(L.P * c.d_ff * 2);
  L.y = take(L.P * c.d_model * 2);
  L.hs = take(c.n_shared > 0 ? L.Tpad * int64_t(c.n_shared) * c.d_ff_shared * 2 : 0);
  L.ys = take(c.n_shared > 0 ? L.Tpad * int64_t(c.d_model) * 2 : 0);
  L.xdev = take(Tm * c.d_model * 2);
  L.outdev = take(Tm * c.d_model * 2);
  // the decode FFN's tile counter and readiness counters
  L.ffn_ctr = take(ffn_counter_bytes());
  // the FP8 path: E4M3 codes of the permuted rows, of x, of H and Hs, each with its scale atoms
  // (512 bytes per 128 rows and 128 columns)
  L.Pa = (L.P + 127) / 128 * 128;
  if (c.flags & MOE_FLAG_FP8) {
    const int64_t d = c.d_model, I = c.d_ff, SI = int64_t(c.n_shared) * c.d_ff_shared;
    L.xq_perm = take(size_t(L.Pa) * d);
    L.xs_perm = take(size_t(L.Pa / 128) * (d / 128) * kSfAtomBytes);
    L.xq = take(size_t(L.Tpad) * d);
    L.xs = take(size_t(L.Tpad / 128) * (d / 128) * kSfAtomBytes);
    L.hq = take(size_t(L.Pa) * I);
    L.hs_perm = take(size_t(L.Pa / 128) * (I / 128) * kSfAtomBytes);
    L.hsq = take(size_t(L.Tpad) * SI);
    L.hss = take(size_t(L.Tpad / 128) * (SI / 128) * kSfAtomBytes);
  }
  L.total = o;
  return L;
}

// The backward's buffers: K-major copies of the expert weights for its two data-gradient GEMMs, the
// recompute's [da | db] rows, the gate gradient's partial sums, the router's dz and dz E, and the
// per-segment partial sums of dE.
constexpr int kDeMaxSegments = 16;
struct BwdLayout {
  size_t wdT, wguT, swdT, swguT, dab, dabs, dg_part, dz, dxr, de_part, dgate;
  // the router's GEMM operands: logits, dz in bf16, K-range tables
  size_t zf, dzb, rt_kstart, rt_kcount;
  int64_t Npad;
  // the weight gradients' operands (row-major, read MN-major by the GEMMs): g dh and m per routed row,
  // m per token of the shared experts
  size_t dy, mrows, msrows, sh_kstart, sh_kcount, total;
};

BwdLayout make_bwd_layout(const moe_config& c, const Layout& L) {
  BwdLayout B{};
  const int64_t N = c.n_routed, I = c.d_ff, d = c.d_model, Ks = c.n_shared, Is = c.d_ff_shared;
  const int64_t Tm = c.max_tokens, Km = c.max_k;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  B.wdT = take(size_t(N) * I * d * 2);
  B.wguT = take(size_t(N) * d * 2 * I * 2);
  B.swdT = take(size_t(Ks) * Is * d * 2);
  B.swguT = take(size_t(Ks) * d * 2 * Is * 2);
  B.dab = take(size_t(L.P) * 2 * I * 2);
  B.dabs = take(size_t(L.Tpad) * Ks * 2 * Is * 2);
  B.dg_part = take(size_t(L.P) * ceil_div(I, kGuBN / 2) * 4);
  B.dz = take(size_t(Tm) * N * 4);
  B.dxr = take(size_t(Tm) * d * 4);
  B.de_part = take(size_t(kDeMaxSegments) * N * d * 4);
  B.dgate = take(size_t(Tm) * Km * 4);
  B.Npad = (N + 15) / 16 * 16;
  B.zf = take(size_t(Tm) * B.Npad * 4);
  B.dzb = take(size_t(Tm) * B.Npad * 2);
  B.rt_kstart = take(kDeMaxSegments * 4);
  B.rt_kcount = take(kDeMaxSegments * 4);
  B.dy = take(size_t(L.P) * d * 2);
  B.mrows = take(size_t(L.P) * I * 2);
  B.msrows = take(size_t(L.Tpad) * Ks * Is * 2);
  B.sh_kstart = take(64 * 4);
  B.sh_kcount = take(64 * 4);
  B.total = o;
  return B;
}

moe_status check_config(const moe_config* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->gate != MOE_GATE_SOFTMAX && c->gate != MOE_GATE_SIGMOID_BIASED) return MOE_ERR_INVALID_ARG;
  if (c->n_routed < 1 || c->max_k < 1 || c->max_tokens < 1 || c->n_shared < 0) return MOE_ERR_SHAPE;
  if (c->d_model < 16 || c->d_ff < 16 || (c->n_shared > 0 && c->d_ff_shared < 16)) return MOE_ERR_SHAPE;
  if (c->max_tokens > kMaxTokens || c->d_model > 65536 || c->d_ff > 65536 || c->d_ff_shared > 65536 ||
      c->n_shared > 64)
    return MOE_ERR_SHAPE;
  if (c->n_routed > kMaxRouted || c->max_k > kMaxK) return MOE_ERR_UNSUPPORTED;
  if (c->max_k > c->n_routed) return MOE_ERR_INVALID_ARG;
  if (c->d_model % 16 || c->d_ff % 16 || (c->n_shared > 0 && c->d_ff_shared % 16)) return MOE_ERR_ALIGNMENT;
  const uint32_t known =
      MOE_FLAG_NO_RESIDUAL | MOE_FLAG_NO_SHARED | MOE_FLAG_NO_ROUTED | MOE_FLAG_FP8 | MOE_FLAG_DEBUG_WAIT_TIMEOUT;
  if (c->flags & ~known) return MOE_ERR_INVALID_ARG;
  if ((c->flags & MOE_FLAG_FP8) && (c->d_model % 128 || c->d_ff % 128 || (c->n_shared > 0 && c->d_ff_shared % 128)))
    return MOE_ERR_ALIGNMENT;
  if ((c->flags & MOE_FLAG_FP8) && (c->d_model > 8192 || c->d_ff > 8192 || c->d_ff_shared > 8192))
    return MOE_ERR_SHAPE;  // at most 64 scale groups along a GEMM's K
  if (c->ep_ranks > 1) {
    if (c->ep_ranks > kEpMaxRanks || c->n_routed % c->ep_ranks || c->ep_rank < 0 || c->ep_rank >= c->ep_ranks)
      return MOE_ERR_INVALID_ARG;
  } else if (c->ep_ranks < 0 || c->ep_rank != 0) {
    return MOE_ERR_INVALID_ARG;
  }
  if (c->route_nodes != 0 || c->route_max_nodes != 0) {
    if (c->route_nodes < 1 || c->route_nodes > kMaxRouteNodes || c->n_routed % c->route_nodes ||
        c->route_max_nodes < 1 || c->route_max_nodes > c->route_nodes ||
        c->max_k > c->route_max_nodes * (c->n_routed / c->route_nodes))
      return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || !na || !nb) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

class DeviceGuard {
 public:
  explicit DeviceGuard(int dev) {
    cudaGetDevice(&prev_);
    if (prev_ != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() { cudaSetDevice(prev_); }

 private:
  int prev_ = 0;
};

}  // namespace

struct moe_ctx {
  moe_config cfg;
  int device = 0;
  int num_sms = 148;
  int max_pairs = 74;  // co-resident CTA pairs of the GEMM kernel (clusters live within one GPC)
  Layout L;
  uint8_t* ws = nullptr;
  cudaStream_t last_stream = nullptr;
  int64_t last_T = 0;
  int last_K = 0;
  // TMA descriptors: workspace ones are fixed, the others follow the caller's pointers
  CUtensorMap tm_xperm, tm_h, tm_hs;
  CUtensorMap tm_xperm32, tm_h32, tm_hs32;  // 32-row token boxes of the decode FFN
  CUtensorMap tm_xq_perm, tm_xq, tm_hq, tm_hsq;  // FP8 codes of the activations (128-row boxes)
  CUtensorMap tm_xq_perm32, tm_xq32, tm_hq32, tm_hsq32;  // the same with 32-row boxes (FP8 decode FFN)
  MapCache tm8_wg, tm8_wu, tm8_wd, tm8_swg, tm8_swu, tm8_swd;  // FP8 weight codes
  MapCache tm8_wd128, tm8_swd128;  // W_down codes with 128-row boxes (FP8 decode FFN)
  MapCache tm_x, tm_x32, tm_router, tm_wg, tm_wu, tm_wd, tm_swg, tm_swu, tm_swd;
  // host-buffer forward: copy streams and per-chunk events, created on first use
  cudaStream_t copy_in = nullptr, copy_out = nullptr;
  cudaEvent_t host_start = nullptr, in_done[kHostChunks] = {}, fwd_done[kHostChunks] = {};
  bool host_ready = false;  // all of the above created
  // per-kernel timing: event pairs recorded around each launch while enabled
  uint32_t timing_mask = 0;  // bit k: time kernel k
  std::vector<cudaEvent_t> ev_pool[MOE_KERNEL_COUNT];
  size_t ev_used[MOE_KERNEL_COUNT] = {};
  // expert parallelism: the ranks' workspaces, which of them this handle opened, the
  // forward's tokens and its step (1 routed, 2 dispatched, 3 experts done, 4 combined)
  EpPeers peers{};
  bool peers_set = false;
  bool ipc_opened[kEpMaxRanks] = {};
  const void* ep_x = nullptr;
  int64_t ep_T = 0;
  int ep_K = 0;
  int ep_stage = 0;
  // the last forward: 1 moe_forward (the backward may follow), 0 anything else
  int last_forward = 0;
  // the backward's own buffers (allocated by its first call) and their descriptors
  uint8_t* bws = nullptr;
  CUtensorMap tm_b_dhperm, tm_b_wdT, tm_b_swdT, tm_b_dab, tm_b_wguT, tm_b_dabs, tm_b_swguT;
  CUtensorMap tm_w_dy, tm_w_m, tm_w_dab, tm_w_xperm, tm_w_ms, tm_w_dabs;  // 64 x 64 MN-major boxes
  CUtensorMap tm_b_dzb;
  MapCache tm_b_dh, tm_b_E, tm_w_dh, tm_w_x, tm_w_E, tm_w_dzb;

  template <typename T>
  T* at(size_t off) const {
    return reinterpret_cast<T*>(ws + off);
  }
};

namespace {

// Batches up to this size launch every kernel of the forward with
// programmatic stream serialization: a kernel may be scheduled while the one
// before it drains, runs its prologue, and waits (griddepcontrol.wait) before
// touching memory that another kernel writes.  Small forwards are bound by
// launch and ramp latency and gain from the overlap (16B decode, T = 32:
// 0.194 -> 0.185 ms); large ones run at the power cap, where it gained nothing
// (16B prefill: 2.234 -> 2.264 ms), so they launch plainly.
constexpr int64_t kPdlMaxT = 512;

// cluster > 1 launches clusters of that many CTAs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster,
                       bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int K>
cudaError_t launch_router_k(bool sigmoid, dim3 grid, size_t smem, cudaStream_t s, bool pdl, const CUtensorMap& tx,
                            const CUtensorMap& te, const RouterArgs& ra) {
  const dim3 b(kRouterThreads);
  if (ra.nodes > 0)
    return sigmoid ? launch_pdl(router_topk_kernel<K, true, true>, grid, b, smem, s, 1, pdl, tx, te, ra)
                   : launch_pdl(router_topk_kernel<K, false, true>, grid, b, smem, s, 1, pdl, tx, te, ra);
  return sigmoid ? launch_pdl(router_topk_kernel<K, true, false>, grid, b, smem, s, 1, pdl, tx, te, ra)
                 : launch_pdl(router_topk_kernel<K, false, false>, grid, b, smem, s, 1, pdl, tx, te, ra);
}

cudaError_t launch_router(int K, bool sigmoid, dim3 grid, size_t smem, cudaStream_t s, bool pdl,
                          const CUtensorMap& tx, const CUtensorMap& te, const RouterArgs& ra) {
  switch (K) {
    case 1: return launch_router_k<1>(sigmoid, grid, smem, s, pdl, tx, te, ra);
    case 2: return launch_router_k<2>(sigmoid, grid, smem, s, pdl, tx, te, ra);
    case 3: return launch_router_k<3>(sigmoid, grid, smem, s, pdl, tx, te, ra);
    case 4: return launch_router_k<4>(sigmoid, grid, smem, s, pdl, tx, te, ra);
    case 5: return launch_router_k<5>(sigmoid, grid, smem, s, pdl, tx, te, ra);
    case 6: return launch_router_k<6>(sigmoid, grid, smem, s, pdl, tx, te, ra);
    case 7: return launch_router_k<7>(sigmoid, grid, smem, s, pdl, tx, te, ra);
    default: return launch_router_k<8>(sigmoid, grid, smem, s, pdl, tx, te, ra);
  }
}

template <int K>
cudaError_t set_router_attrs_k(size_t smem) {
  const int sm = static_cast<int>(smem);
  const auto attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(router_topk_kernel<K, true, false>, attr, sm)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(router_topk_kernel<K, false, false>, attr, sm)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(router_topk_kernel<K, true, true>, attr, sm)) != cudaSuccess) return e;
  return cudaFuncSetAttribute(router_topk_kernel<K, false, true>, attr, sm);
}

cudaError_t set_kernel_attrs() {
  const size_t rs = router_smem_bytes(256);
  cudaError_t e = cudaSuccess;
  if ((e = set_router_attrs_k<1>(rs)) != cudaSuccess) return e;
  if ((e = set_router_attrs_k<2>(rs)) != cudaSuccess) return e;
  if ((e = set_router_attrs_k<3>(rs)) != cudaSuccess) return e;
  if ((e = set_router_attrs_k<4>(rs)) != cudaSuccess) return e;
  if ((e = set_router_attrs_k<5>(rs)) != cudaSuccess) return e;
  if ((e = set_router_attrs_k<6>(rs)) != cudaSuccess) return e;
  if ((e = set_router_attrs_k<7>(rs)) != cudaSuccess) return e;
  if ((e = set_router_attrs_k<8>(rs)) != cudaSuccess) return e;
  const int us = static_cast<int>(gateup_smem_bytes());
  if ((e = cudaFuncSetAttribute(gateup_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, us))) return e;
  if ((e = cudaFuncSetAttribute(gateup_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, us))) return e;
  const int gs = static_cast<int>(gemm_smem_bytes());
  if ((e = cudaFuncSetAttribute(down_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, gs))) return e;
  if ((e = cudaFuncSetAttribute(decode_ffn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(ffn_smem_bytes()))))
    return e;
  const int fs = static_cast<int>(fp8_gemm_smem_bytes());
  if ((e = cudaFuncSetAttribute(fp8_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, fs))) return e;
  if ((e = cudaFuncSetAttribute(fp8_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, fs))) return e;
  return cudaFuncSetAttribute(decode_ffn8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(ffn8_smem_bytes()));
}

bool refresh_u8(MapCache& c, const void* p, uint64_t d2, uint64_t rows, uint64_t cols, uint32_t box_rows, int rank) {
  if (c.ptr == p) return true;
  if (!encode_u8(&c.map, p, d2, rows, cols, box_rows, rank)) {
    c.ptr = nullptr;
    return false;
  }
  c.ptr = p;
  c.rows = 0;
  return true;
}

// Re-encode a cached descriptor when the caller's pointer (or row count) changes.
bool refresh(MapCache& c, const void* p, int64_t rows_key, uint64_t d2, uint64_t rows, uint64_t cols,
             uint32_t box_rows, int rank) {
  if (c.ptr == p && c.rows == rows_key) return true;
  if (!encode_bf16(&c.map, p, d2, rows, cols, box_rows, rank)) {
    c.ptr = nullptr;
    return false;
  }
  c.ptr = p;
  c.rows = rows_key;
  return true;
}

// Launch `pairs` CTA pairs (clusters of 2) of the down GEMM kernel.
cudaError_t launch_down(int pairs, cudaStream_t s, bool pdl, const CUtensorMap& A, const CUtensorMap& B,
                        const CUtensorMap& As, const CUtensorMap& Bs, const GemmArgs& ga) {
  return launch_pdl(down_gemm_kernel, dim3(2 * pairs), dim3(kGemmThreads), gemm_smem_bytes(), s, 2, pdl, A, B, As, Bs,
                    ga);
}


cudaError_t launch_gateup(int ctas, cudaStream_t s, bool pdl, const CUtensorMap& A, const CUtensorMap& G,
                          const CUtensorMap& U, const CUtensorMap& As, const CUtensorMap& Gs, const CUtensorMap& Us,
                          const GateUpArgs& ga, bool backward = false) {
  return backward ? launch_pdl(gateup_gemm_kernel<true>, dim3(ctas), dim3(kGuThreads), gateup_smem_bytes(), s, 1, pdl,
                               A, G, U, As, Gs, Us, ga)
                  : launch_pdl(gateup_gemm_kernel<false>, dim3(ctas), dim3(kGuThreads), gateup_smem_bytes(), s, 1, pdl,
                               A, G, U, As, Gs, Us, ga);
}

// Destroys the host-buffer forward's copy streams and events (those that exist).
void release_host_pipeline(moe_ctx* h) {
  if (h->copy_in) cudaStreamDestroy(h->copy_in);
  if (h->copy_out) cudaStreamDestroy(h->copy_out);
  if (h->host_start) cudaEventDestroy(h->host_start);
  h->copy_in = h->copy_out = nullptr;
  h->host_start = nullptr;
  for (int c = 0; c < kHostChunks; ++c) {
    if (h->in_done[c]) cudaEventDestroy(h->in_done[c]);
    if (h->fwd_done[c]) cudaEventDestroy(h->fwd_done[c]);
    h->in_done[c] = h->fwd_done[c] = nullptr;
  }
  h->host_ready = false;
}

// Records a start/stop event pair around one launch when timing is enabled.
class KernelTimer {
 public:
  KernelTimer(moe_ctx* h, int id, cudaStream_t s) : h_(h), id_(id), s_(s) {
    if (!((h_->timing_mask >> id_) & 1u)) return;
    auto& pool = h_->ev_pool[id_];
    size_t& used = h_->ev_used[id_];
    while (pool.size() < used + 2) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return;
      pool.push_back(e);
    }
    stop_ = pool[used + 1];
    cudaEventRecord(pool[used], s_);
    used += 2;
  }
  ~KernelTimer() {
    if (stop_) cudaEventRecord(stop_, s_);
  }

 private:
  moe_ctx* h_;
  int id_;
  cudaStream_t s_;
  cudaEvent_t stop_ = nullptr;
};

PermuteArgs permute_args(moe_ctx* h, const void* x, int64_t T, int32_t K, const RouterArgs& ra, bool gather);

// The router step shared by the bf16 and FP8 forwards: affinities, top-K, the
// per-block expert histogram and the scan (router_topk.cuh).  Records the
// call's stream, T and K for moe_get_routing / moe_status_query.  fused > 0:
// route_permute_decode_kernel, which also forms the permutation (fused == 2:
// with the row copies); the caller launches no permutation then.
moe_status enqueue_router(moe_ctx* h, const void* x, int64_t T, const moe_router* router, int32_t K,
                          cudaStream_t s0, bool pdl, RouterArgs& ra, int fused = 0) {
  const moe_config& c = h->cfg;
  const Layout& L = h->L;
  const int64_t d = c.d_model, N = c.n_routed;
  const bool sigmoid = c.gate == MOE_GATE_SIGMOID_BIASED;
  const int Npad = ((int)N + 15) / 16 * 16;
  static_assert(kGuBoxRowsA == kRouterBM, "x serves as A of the router and of the shared gate/up GEMM");
  if (!refresh(h->tm_x, x, T, 1, T, d, kGuBoxRowsA, 2) ||
      !refresh(h->tm_router, router->weight, 0, 1, N, d, (uint32_t)Npad, 2))
    return MOE_ERR_CUDA;
  h->last_stream = s0;
  h->last_T = T;
  h->last_K = K;
  const int nblk = ceil_div(T, 128);
  ra = RouterArgs{};
  ra.T = (int)T;
  ra.N = (int)N;
  ra.Npad = Npad;
  ra.num_kb = ceil_div(d, kBK);
  ra.nblk = nblk;
  ra.tmem_cols = Npad <= 32 ? 32u : Npad <= 64 ? 64u : Npad <= 128 ? 128u : 256u;
  ra.logit_bias = router->logit_bias;
  ra.select_bias = router->select_bias;
  ra.idx = h->at<int32_t>(L.idx);
  ra.gate = h->at<float>(L.gate);
  ra.block_counts = h->at<int32_t>(L.bc);
  ra.counts = h->at<int32_t>(L.counts);
  ra.offsets = h->at<int32_t>(L.offsets);
  ra.row_start = h->at<int32_t>(L.row_start);
  ra.mtile_start = h->at<int32_t>(L.mtile);
  ra.mtile128_start = h->at<int32_t>(L.mtile128);
  ra.done_counter = h->at<uint32_t>(L.done);
  ra.err = h->at<uint32_t>(L.err);
  ra.timeout_ns = kTimeoutNs;
  if (c.route_nodes > 0) {
    ra.nodes = c.route_nodes;
    ra.per_node = (int)(N / c.route_nodes);
    ra.max_nodes = c.route_max_nodes;
  }
  KernelTimer kt(h, MOE_KERNEL_ROUTER, s0);
  if (fused > 0) {
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    const __nv_bfloat16* eb = static_cast<const __nv_bfloat16*>(router->weight);
    const PermuteArgs pa = permute_args(h, x, T, K, ra, fused == 2);
    const RouteTables rt{ra.counts, ra.offsets, ra.row_start, ra.mtile_start, ra.mtile128_start, ra.block_counts};
    const dim3 grid((unsigned)(T * kRouteCluster)), block(kRouteThreads);
    const cudaError_t e =
        sigmoid ? launch_pdl(route_permute_decode_kernel<true>, grid, block, 0, s0, 1, pdl, xb, eb, ra, pa, rt)
                : launch_pdl(route_permute_decode_kernel<false>, grid, block, 0, s0, 1, pdl, xb, eb, ra, pa, rt);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  if (T <= kSmallRouterMaxT) {
    // a few tokens: one CTA per token on the CUDA cores
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    const __nv_bfloat16* eb = static_cast<const __nv_bfloat16*>(router->weight);
    SmallRouterArgs sa{h->at<float>(L.small_logits), h->at<uint32_t>(L.tok_done)};
    const dim3 grid((unsigned)T, (unsigned)ceil_div(N, kSmallRouterGroup)), block(kSmallRouterThreads);
    const cudaError_t e =
        sigmoid ? launch_pdl(router_small_kernel<true>, grid, block, 0, s0, 1, pdl, xb, eb, (int)d, K, ra, sa)
                : launch_pdl(router_small_kernel<false>, grid, block, 0, s0, 1, pdl, xb, eb, (int)d, K, ra, sa);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  const size_t smem = router_smem_bytes(Npad);
  return launch_router(K, sigmoid, dim3(nblk), smem, s0, pdl, h->tm_x.map, h->tm_router.map, ra) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

// The permutation's arguments (permute.cuh), shared by both forwards.
PermuteArgs permute_args(moe_ctx* h, const void* x, int64_t T, int32_t K, const RouterArgs& ra, bool gather) {
  const Layout& L = h->L;
  const int nblk = ceil_div(T, 128);
  PermuteArgs pa{};
  pa.T = (int)T;
  pa.K = K;
  pa.N = h->cfg.n_routed;
  pa.d = h->cfg.d_model;
  const int split = (4 * h->num_sms + nblk - 1) / nblk;
  // CTAs per 128-token block for the row copies: about four per SM in all (16B prefill, T = 16384:
  // 0.110 -> 0.100 ms against two), at most 8, or 32 for batches of up to 4 blocks (a 32-token decode
  // batch copies one token row per CTA: 16B decode permutation 10.2 -> 8.6 us; more than 8 measured
  // slower on the V3 layer, T = 4096)
  const int max_split = nblk <= 4 ? 32 : 8;
  pa.split = split < 1 ? 1 : split > max_split ? max_split : split;
  pa.idx = ra.idx;
  pa.gate = ra.gate;
  pa.block_base = ra.block_counts;
  pa.offsets = ra.offsets;
  pa.row_start = ra.row_start;
  pa.src = h->at<int32_t>(L.src);
  pa.slot_of = h->at<int32_t>(L.slot);
  pa.gate_perm = h->at<float>(L.gate_perm);
  pa.x = static_cast<const __nv_bfloat16*>(x);
  pa.x_perm = h->at<__nv_bfloat16>(L.x_perm);
  pa.gather = gather ? 1 : 0;
  pa.tile_ctr = h->at<int>(L.tile_ctr);
  return pa;
}

// The final sum (combine_kernel): one warp per (token, chunk of a row): whole
// rows once the batch alone gives every SM a full load of warps, shorter
// chunks (>= 256 columns) below that (V3 layer, T = 4096, d = 7168: 0.272 ->
// 0.223 ms).
moe_status launch_combine(moe_ctx* h, const CombineArgs& ca, int64_t T, int64_t d, cudaStream_t s0, bool pdl) {
  KernelTimer kt(h, MOE_KERNEL_COMBINE, s0);
  const int64_t resident = int64_t(h->num_sms) * 64;  // warps the SMs hold at once
  int cols = (int)d;
  if (T < resident) {
    const int chunks = ceil_div(2 * resident, T);
    cols = ceil_div(ceil_div(d, chunks), 256) * 256;
  }
  const int64_t warps = T * ceil_div(d, cols);
  if (launch_pdl(combine_kernel, dim3(ceil_div(warps * 32, 256)), dim3(256), 0, s0, 1, pdl, ca, cols) != cudaSuccess)
    return MOE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// The routed experts' tables of the grouped GEMMs (device pointers; G = 0: no routed tiles).
struct ExpertTables {
  int G;                     // routed experts (groups of the row buffer)
  const int32_t* mtile128;   // [G + 1] prefix of ceil(rows / 128): the gate/up GEMM's m-tiles
  const int32_t* mtile;      // [G + 1] prefix of ceil(rows / 256): the down GEMM's pair tiles
  const int32_t* row_start;  // [G + 1] first row of each expert in X_perm, H and Y
  const float* row_scale;    // the gate of each row
};

// The expert GEMMs of a batch above the decode size, on the weight maps of the
// handle: gate/up + SwiGLU, then down + gate scale, each one persistent launch
// with the shared experts' tiles (the T rows of x) first and then the routed
// experts' (tables on the device).
moe_status enqueue_expert_gemms(moe_ctx* h, int64_t T, bool do_shared, const ExpertTables& et, int* tile_ctr,
                                cudaStream_t s0, bool pdl) {
  const moe_config& c = h->cfg;
  const Layout& L = h->L;
  const int64_t d = c.d_model, I = c.d_ff, Ks = c.n_shared, Is = c.d_ff_shared;
  const bool do_routed = et.G > 0;
  const int num_kb = ceil_div(d, kGuBK);
  GateUpArgs g{};
  if (do_routed) {
    g.num_groups = et.G;
    g.mtile_start = et.mtile128;
    g.row_start = et.row_start;
    g.n_tiles = ceil_div(I, kGuBN / 2);
    g.n_limit = (int)I;
    g.out = h->at<__nv_bfloat16>(L.h);
    g.ld_out = (int)I;
  }
  if (do_shared) {
    g.sh_rows = (int)T;
    g.sh_n_tiles = ceil_div(Ks * Is, kGuBN / 2);
    g.sh_n_limit = (int)(Ks * Is);
    g.sh_out = h->at<__nv_bfloat16>(L.hs);
    g.sh_ld_out = (int)(Ks * Is);
  }
  g.num_kb = num_kb;
  g.tile_ctr = tile_ctr;
  g.die_split = h->num_sms / 2;
  g.err = h->at<uint32_t>(L.err);
  g.timeout_ns = kTimeoutNs;
  g.debug_wait = (c.flags & MOE_FLAG_DEBUG_WAIT_TIMEOUT) ? 1 : 0;
  // with routed tiles the count is known only on the device: one CTA per SM
  const int sh_tiles = do_shared ? ceil_div(T, kGuBM) * g.sh_n_tiles : 0;
  const int ctas = do_routed || sh_tiles > h->num_sms ? h->num_sms : sh_tiles;
  // an absent part's maps are never read; the present part's stand in
  const CUtensorMap& sA = do_shared ? h->tm_x.map : h->tm_xperm;
  const CUtensorMap& sG = do_shared ? h->tm_swg.map : h->tm_wg.map;
  const CUtensorMap& sU = do_shared ? h->tm_swu.map : h->tm_wu.map;
  {
    KernelTimer kt(h, MOE_KERNEL_GATE_UP, s0);
    if (launch_gateup(ctas, s0, pdl, h->tm_xperm, h->tm_wg.map, h->tm_wu.map, sA, sG, sU, g) != cudaSuccess)
      return MOE_ERR_CUDA;
  }

  GemmArgs g2{};
  if (do_routed) {
    g2.num_groups = et.G;
    g2.mtile_start = et.mtile;
    g2.row_start = et.row_start;
    g2.num_kb = ceil_div(I, kGemmBK);
    g2.row_scale = et.row_scale;
    g2.out = h->at<__nv_bfloat16>(L.y);
  }
  if (do_shared) {
    g2.sh_rows = (int)T;
    g2.sh_num_kb = ceil_div(Is, kGemmBK);
    g2.sh_J = (int)Ks;
    g2.sh_k_per_j = (int)Is;
    g2.sh_out = h->at<__nv_bfloat16>(L.ys);
  }
  g2.n_tiles = ceil_div(d, kGemmBN);
  g2.n_limit = (int)d;
  g2.ld_out = (int)d;
  g2.err = h->at<uint32_t>(L.err);
  g2.timeout_ns = kTimeoutNs;
  const int sh_tiles2 = do_shared ? ceil_div(T, kGemmBM) * g2.n_tiles : 0;
  const int pairs = do_routed || sh_tiles2 > h->max_pairs ? h->max_pairs : sh_tiles2;
  const CUtensorMap& sA2 = do_shared ? h->tm_hs : h->tm_h;
  const CUtensorMap& sB2 = do_shared ? h->tm_swd.map : h->tm_wd.map;
  KernelTimer kt(h, MOE_KERNEL_DOWN, s0);
  if (launch_down(pairs, s0, pdl, h->tm_h, h->tm_wd.map, sA2, sB2, g2) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

// The FP8 layer's expert GEMMs (fp8_gemm.cuh): gate/up with SwiGLU and H's quantization, then down with the
// gate scale; the shared experts' tiles over the T rows of x's codes first, then the routed experts' (G groups,
// tables on the device; G = 0: none).  The FP8 weight maps of the handle must hold the caller's pointers.
moe_status enqueue_fp8_expert_gemms(moe_ctx* h, int64_t T, bool do_shared, int G, const int32_t* mtile128,
                                    const int32_t* row_start, const moe_experts_fp8* experts,
                                    const moe_experts_fp8* shared, cudaStream_t s0, bool pdl) {
  const moe_config& c = h->cfg;
  const Layout& L = h->L;
  const int64_t d = c.d_model, I = c.d_ff, Ks = c.n_shared, Is = c.d_ff_shared;
  const bool do_routed = G > 0;
  const int64_t SI = Ks * Is;
  // an absent part's maps are never read; the present part's stand in
  const CUtensorMap& A = do_routed ? h->tm_xq_perm : h->tm_xq;
  const CUtensorMap& As = do_shared ? h->tm_xq : h->tm_xq_perm;
  const CUtensorMap& Wg = do_routed ? h->tm8_wg.map : h->tm8_swg.map;
  const CUtensorMap& Wu = do_routed ? h->tm8_wu.map : h->tm8_swu.map;
  const CUtensorMap& Wgs = do_shared ? h->tm8_swg.map : h->tm8_wg.map;
  const CUtensorMap& Wus = do_shared ? h->tm8_swu.map : h->tm8_wu.map;
  Fp8GemmArgs g{};
  if (do_routed) {
    g.num_groups = G;
    g.mtile_start = mtile128;
    g.row_start = row_start;
    g.n_tiles = ceil_div(I, kF8BN / 2);
    g.num_kg = (int)(d / kF8BK);
    g.a_atoms = h->at<uint8_t>(L.xs_perm);
    g.a_groups = (int)(d / kF8BK);
    g.w_scale0 = experts->s_gate;
    g.w_scale1 = experts->s_up;
    g.w_rows128 = (int)(I / 128);
    g.hq = h->at<uint8_t>(L.hq);
    g.hs_atoms = h->at<uint8_t>(L.hs_perm);
    g.h_groups = (int)(I / kF8BK);
    g.ld_out = (int)I;
    g.n_limit = (int)I;
  }
  if (do_shared) {
    g.sh_rows = (int)T;
    g.sh_n_tiles = ceil_div(SI, kF8BN / 2);
    g.sh_J = 1;
    g.sh_kg_per_j = (int)(d / kF8BK);
    g.sh_a_atoms = h->at<uint8_t>(L.xs);
    g.sh_a_groups = (int)(d / kF8BK);
    g.sh_w_scale0 = shared->s_gate;
    g.sh_w_scale1 = shared->s_up;
    g.sh_w_rows128 = (int)(Is / 128);
    g.sh_hq = h->at<uint8_t>(L.hsq);
    g.sh_hs_atoms = h->at<uint8_t>(L.hss);
    g.sh_h_groups = (int)(SI / kF8BK);
    g.sh_ld_out = (int)SI;
    g.sh_n_limit = (int)SI;
  }
  g.err = h->at<uint32_t>(L.err);
  g.timeout_ns = kTimeoutNs;
  g.debug_wait = (c.flags & MOE_FLAG_DEBUG_WAIT_TIMEOUT) ? 1 : 0;
  const int sh_tiles = do_shared ? ceil_div(T, kF8BM) * g.sh_n_tiles : 0;
  const int ctas = do_routed || sh_tiles > h->num_sms ? h->num_sms : sh_tiles;
  {
    KernelTimer kt(h, MOE_KERNEL_GATE_UP, s0);
    if (launch_pdl(fp8_gemm_kernel<true>, dim3(ctas), dim3(kF8Threads), fp8_gemm_smem_bytes(), s0, 1, pdl, A, Wg,
                   Wu, As, Wgs, Wus, g) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  const CUtensorMap& HA = do_routed ? h->tm_hq : h->tm_hsq;
  const CUtensorMap& HAs = do_shared ? h->tm_hsq : h->tm_hq;
  const CUtensorMap& Wd = do_routed ? h->tm8_wd.map : h->tm8_swd.map;
  const CUtensorMap& Wds = do_shared ? h->tm8_swd.map : h->tm8_wd.map;
  Fp8GemmArgs g2{};
  if (do_routed) {
    g2.num_groups = G;
    g2.mtile_start = mtile128;
    g2.row_start = row_start;
    g2.n_tiles = ceil_div(d, kF8BN);
    g2.num_kg = (int)(I / kF8BK);
    g2.a_atoms = h->at<uint8_t>(L.hs_perm);
    g2.a_groups = (int)(I / kF8BK);
    g2.w_scale0 = experts->s_down;
    g2.w_rows128 = (int)(d / 128);
    g2.row_scale = h->at<float>(L.gate_perm);
    g2.y = h->at<__nv_bfloat16>(L.y);
    g2.ld_out = (int)d;
    g2.n_limit = (int)d;
  }
  if (do_shared) {
    g2.sh_rows = (int)T;
    g2.sh_n_tiles = ceil_div(d, kF8BN);
    g2.sh_J = (int)Ks;
    g2.sh_kg_per_j = (int)(Is / kF8BK);
    g2.sh_k_per_j = (int)Is;
    g2.sh_a_atoms = h->at<uint8_t>(L.hss);
    g2.sh_a_groups = (int)(SI / kF8BK);
    g2.sh_w_scale0 = shared->s_down;
    g2.sh_w_rows128 = (int)(d / 128);
    g2.sh_y = h->at<__nv_bfloat16>(L.ys);
    g2.sh_ld_out = (int)d;
    g2.sh_n_limit = (int)d;
  }
  g2.err = h->at<uint32_t>(L.err);
  g2.timeout_ns = kTimeoutNs;
  const int sh_tiles2 = do_shared ? ceil_div(T, kF8BM) * g2.sh_n_tiles : 0;
  const int ctas2 = do_routed || sh_tiles2 > h->num_sms ? h->num_sms : sh_tiles2;
  KernelTimer kt(h, MOE_KERNEL_DOWN, s0);
  if (launch_pdl(fp8_gemm_kernel<false>, dim3(ctas2), dim3(kF8Threads), fp8_gemm_smem_bytes(), s0, 1, pdl, HA, Wd,
                 Wd, HAs, Wds, Wds, g2) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_SHAPE: return "MOE_ERR_SHAPE";
    case MOE_ERR_ALIGNMENT: return "MOE_ERR_ALIGNMENT";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_NOMEM: return "MOE_ERR_NOMEM";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
  }
  return "MOE_ERR_UNKNOWN";
}

moe_status moe_workspace_bytes(const moe_config* cfg, uint64_t* bytes) {
  if (!bytes) return MOE_ERR_INVALID_ARG;
  const moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  *bytes = make_layout(*cfg).total;
  return MOE_OK;
}

moe_status moe_create(const moe_config* cfg, int device, moe_handle* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return MOE_ERR_CUDA;
  if (prop.major != 10) return MOE_ERR_UNSUPPORTED;
  if (!load_encode()) return MOE_ERR_CUDA;
  DeviceGuard guard(device);
  if (set_kernel_attrs() != cudaSuccess) return MOE_ERR_CUDA;

  moe_ctx* h = new moe_ctx();
  h->cfg = *cfg;
  h->device = device;
  h->num_sms = prop.multiProcessorCount;
  h->L = make_layout(*cfg);
  {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(2 * (prop.multiProcessorCount / 2));
    lc.blockDim = dim3(kGemmThreads);
    lc.dynamicSmemBytes = gemm_smem_bytes();
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, down_gemm_kernel, &lc) != cudaSuccess || clusters < 1) {
      cudaGetLastError();
      delete h;
      return MOE_ERR_CUDA;
    }
    h->max_pairs = clusters < prop.multiProcessorCount / 2 ? clusters : prop.multiProcessorCount / 2;
  }
  if (cudaMalloc(&h->ws, h->L.total) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return MOE_ERR_NOMEM;
  }
  bool ok = cudaMemset(h->ws, 0, align256(4096)) == cudaSuccess;
  ok = ok && cudaMemset(h->ws + h->L.ffn_ctr, 0, ffn_counter_bytes()) == cudaSuccess;
  const moe_config& c = *cfg;
  ok = ok && encode_bf16(&h->tm_xperm, h->ws + h->L.x_perm, 1, h->L.P, c.d_model, kGuBoxRowsA, 2);
  ok = ok && encode_bf16(&h->tm_h, h->ws + h->L.h, 1, h->L.P, c.d_ff, kBoxRowsA, 2);
  ok = ok && encode_bf16(&h->tm_xperm32, h->ws + h->L.x_perm, 1, h->L.P, c.d_model, kFfnBoxRowsX, 2);
  ok = ok && encode_bf16(&h->tm_h32, h->ws + h->L.h, 1, h->L.P, c.d_ff, kFfnBoxRowsX, 2);
  if (c.n_shared > 0) {
    ok = ok && encode_bf16(&h->tm_hs, h->ws + h->L.hs, 1, h->L.Tpad, int64_t(c.n_shared) * c.d_ff_shared, kBoxRowsA, 2);
    ok = ok &&
         encode_bf16(&h->tm_hs32, h->ws + h->L.hs, 1, h->L.Tpad, int64_t(c.n_shared) * c.d_ff_shared, kFfnBoxRowsX, 2);
  }
  if (c.flags & MOE_FLAG_FP8) {
    const int64_t SI = int64_t(c.n_shared) * c.d_ff_shared;
    ok = ok && encode_u8(&h->tm_xq_perm, h->ws + h->L.xq_perm, 1, h->L.Pa, c.d_model, 128, 2);
    ok = ok && encode_u8(&h->tm_xq, h->ws + h->L.xq, 1, h->L.Tpad, c.d_model, 128, 2);
    ok = ok && encode_u8(&h->tm_hq, h->ws + h->L.hq, 1, h->L.Pa, c.d_ff, 128, 2);
    if (SI > 0) ok = ok && encode_u8(&h->tm_hsq, h->ws + h->L.hsq, 1, h->L.Tpad, SI, 128, 2);
    ok = ok && encode_u8(&h->tm_xq_perm32, h->ws + h->L.xq_perm, 1, h->L.Pa, c.d_model, kFfnBoxRowsX, 2);
    ok = ok && encode_u8(&h->tm_xq32, h->ws + h->L.xq, 1, h->L.Tpad, c.d_model, kFfnBoxRowsX, 2);
    ok = ok && encode_u8(&h->tm_hq32, h->ws + h->L.hq, 1, h->L.Pa, c.d_ff, kFfnBoxRowsX, 2);
    if (SI > 0) ok = ok && encode_u8(&h->tm_hsq32, h->ws + h->L.hsq, 1, h->L.Tpad, SI, kFfnBoxRowsX, 2);
  }
  ok = ok && cudaDeviceSynchronize() == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    moe_destroy(h);
    return MOE_ERR_CUDA;
  }
  *out = h;
  return MOE_OK;
}

moe_status moe_forward(moe_handle h, const void* x, int64_t T, const moe_router* router,
                       const moe_experts* experts, const moe_shared* shared, int32_t K, void* out,
                       void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  const moe_config& c = h->cfg;
  if (c.ep_ranks > 1) return MOE_ERR_UNSUPPORTED;
  if (T < 0 || T > c.max_tokens) return MOE_ERR_SHAPE;
  if (K < 1 || K > c.max_k || K > c.n_routed) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;  // nothing to enqueue (an empty tensor may carry a null pointer)
  if (!router || !experts) return MOE_ERR_INVALID_ARG;
  if ((c.n_shared > 0) != (shared != nullptr)) return MOE_ERR_INVALID_ARG;
  if (!x || !out || !router->weight || !experts->w_gate || !experts->w_up || !experts->w_down)
    return MOE_ERR_INVALID_ARG;
  if (shared && (!shared->w_gate || !shared->w_up || !shared->w_down)) return MOE_ERR_INVALID_ARG;
  const bool sigmoid = c.gate == MOE_GATE_SIGMOID_BIASED;
  if (sigmoid ? router->logit_bias != nullptr : router->select_bias != nullptr) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, out, router->weight, router->logit_bias, router->select_bias, experts->w_gate,
                        experts->w_up, experts->w_down, shared ? shared->w_gate : nullptr,
                        shared ? shared->w_up : nullptr, shared ? shared->w_down : nullptr};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_ALIGNMENT;
  const int64_t d = c.d_model, N = c.n_routed, I = c.d_ff, Ks = c.n_shared, Is = c.d_ff_shared;
  const size_t out_bytes = size_t(T) * d * 2;
  const size_t wsz = size_t(N) * I * d * 2, swsz = size_t(Ks) * Is * d * 2;
  if (overlaps(out, out_bytes, x, out_bytes) || overlaps(out, out_bytes, router->weight, size_t(N) * d * 2) ||
      overlaps(out, out_bytes, experts->w_gate, wsz) || overlaps(out, out_bytes, experts->w_up, wsz) ||
      overlaps(out, out_bytes, experts->w_down, wsz) ||
      (shared && (overlaps(out, out_bytes, shared->w_gate, swsz) || overlaps(out, out_bytes, shared->w_up, swsz) ||
                  overlaps(out, out_bytes, shared->w_down, swsz))))
    return MOE_ERR_INVALID_ARG;

  DeviceGuard guard(h->device);
  cudaStream_t s0 = static_cast<cudaStream_t>(stream);
  const Layout& L = h->L;
  const bool do_shared = Ks > 0 && !(c.flags & MOE_FLAG_NO_SHARED);
  const bool do_routed = !(c.flags & MOE_FLAG_NO_ROUTED);

  // descriptors that follow the caller's pointers
  // a decode batch: the weight-streaming FFN, if its token blocks fit the readiness counters
  const bool decode = T <= kDecodeMaxT && decode_token_blocks(T, K, N) <= kFfnMaxBlocks;
  bool ok = true;
  if (decode) ok = ok && refresh(h->tm_x32, x, T, 1, T, d, kFfnBoxRowsX, 2);
  ok = ok && refresh(h->tm_wg, experts->w_gate, 0, N, I, d, kGuBoxRowsB, 3);
  ok = ok && refresh(h->tm_wu, experts->w_up, 0, N, I, d, kGuBoxRowsB, 3);
  ok = ok && refresh(h->tm_wd, experts->w_down, 0, N, d, I, kBoxRowsB, 3);
  if (shared) {
    ok = ok && refresh(h->tm_swg, shared->w_gate, 0, 1, Ks * Is, d, kGuBoxRowsB, 3);
    ok = ok && refresh(h->tm_swu, shared->w_up, 0, 1, Ks * Is, d, kGuBoxRowsB, 3);
    ok = ok && refresh(h->tm_swd, shared->w_down, 0, Ks, d, Is, kBoxRowsB, 3);
  }
  if (!ok) return MOE_ERR_CUDA;

  const bool pdl = T <= kPdlMaxT;
  const int nblk = ceil_div(T, 128);

  // ---- router and permutation ----
  // a decode batch with a small router matrix: both in one launch
  const bool fused_route = decode && route_decode_fits(T, N, d, K);
  RouterArgs ra;
  {
    const moe_status st = enqueue_router(h, x, T, router, K, s0, pdl, ra, fused_route ? (do_routed ? 2 : 1) : 0);
    if (st != MOE_OK) return st;
  }
  PermuteArgs pa = permute_args(h, x, T, K, ra, do_routed);
  if (!fused_route) {
    KernelTimer kt(h, MOE_KERNEL_PERMUTE, s0);
    const dim3 grid(nblk, do_routed ? pa.split : 1);
    if (launch_pdl(permute_gather_kernel, grid, dim3(kPermThreads), 0, s0, 1, pdl, pa) != cudaSuccess)
      return MOE_ERR_CUDA;
  }

  // ---- the expert FFNs of a small batch: one weight-streaming launch (decode_ffn.cuh) ----
  if (decode && (do_routed || do_shared)) {
    FfnArgs f{};
    f.T = (int)T;
    if (do_routed) {
      f.G = (int)N;
      f.n_wb_gu = ceil_div(I, kFfnWB);
      f.n_wb_dn = ceil_div(d, kFfnWB);
      f.kb_gu = ceil_div(d, kFfnBK);
      f.kb_dn = ceil_div(I, kFfnBK);
      f.counts = ra.counts;
      f.row_start = ra.row_start;
      f.row_scale = pa.gate_perm;
      f.h = h->at<__nv_bfloat16>(L.h);
      f.y = h->at<__nv_bfloat16>(L.y);
    }
    if (do_shared) {
      f.sh_blocks = ceil_div(T, kFfnTB);
      f.sh_n_wb_gu = ceil_div(Ks * Is, kFfnWB);
      f.sh_n_wb_dn = ceil_div(d, kFfnWB);
      f.sh_J = (int)Ks;
      f.sh_kb_per_j = ceil_div(Is, kFfnBK);
      f.sh_k_per_j = (int)Is;
      f.hs = h->at<__nv_bfloat16>(L.hs);
      f.ys = h->at<__nv_bfloat16>(L.ys);
    }
    f.kb_gu = ceil_div(d, kFfnBK);  // the shared gate/up tiles' k loop too
    f.I = (int)I;
    f.sh_cols = (int)(Ks * Is);
    f.d = (int)d;
    f.ctr = h->at<uint32_t>(L.ffn_ctr);
    f.err = h->at<uint32_t>(L.err);
    f.timeout_ns = kTimeoutNs;
    f.debug_wait = (c.flags & MOE_FLAG_DEBUG_WAIT_TIMEOUT) ? 1 : 0;
    // an absent part's maps are never read; the present part's stand in
    const CUtensorMap& Wg = do_routed ? h->tm_wg.map : h->tm_swg.map;
    const CUtensorMap& Wu = do_routed ? h->tm_wu.map : h->tm_swu.map;
    const CUtensorMap& Wd = do_routed ? h->tm_wd.map : h->tm_swd.map;
    const CUtensorMap& Xr = do_routed ? h->tm_xperm32 : h->tm_x32.map;
    const CUtensorMap& Hr = do_routed ? h->tm_h32 : h->tm_hs32;
    const CUtensorMap& Wsg = do_shared ? h->tm_swg.map : h->tm_wg.map;
    const CUtensorMap& Wsu = do_shared ? h->tm_swu.map : h->tm_wu.map;
    const CUtensorMap& Wsd = do_shared ? h->tm_swd.map : h->tm_wd.map;
    const CUtensorMap& Hsm = do_shared ? h->tm_hs32 : h->tm_h32;
    KernelTimer kt(h, MOE_KERNEL_GATE_UP, s0);
    if (launch_pdl(decode_ffn_kernel, dim3(h->num_sms), dim3(kFfnThreads), ffn_smem_bytes(), s0, 1, pdl, Wg, Wu, Xr,
                   Wsg, Wsu, h->tm_x32.map, Wd, Hr, Wsd, Hsm, f) != cudaSuccess)
      return MOE_ERR_CUDA;
  }

  // ---- the expert GEMMs: shared experts' tiles first, then the routed experts' ----
  if (!decode && (do_routed || do_shared)) {
    ExpertTables et{};
    if (do_routed) et = ExpertTables{(int)N, ra.mtile128_start, ra.mtile_start, ra.row_start, pa.gate_perm};
    const moe_status st = enqueue_expert_gemms(h, T, do_shared, et, pa.tile_ctr, s0, pdl);
    if (st != MOE_OK) return st;
  }

  // ---- the final sum ----
  h->last_forward = 1;
  CombineArgs ca{};
  ca.T = (int)T;
  ca.K = K;
  ca.d = (int)d;
  ca.x = static_cast<const __nv_bfloat16*>(x);
  ca.ys = do_shared ? h->at<__nv_bfloat16>(L.ys) : nullptr;
  ca.y = h->at<__nv_bfloat16>(L.y);
  ca.slot_of = pa.slot_of;
  ca.out = static_cast<__nv_bfloat16*>(out);
  ca.add_residual = (c.flags & MOE_FLAG_NO_RESIDUAL) ? 0 : 1;
  ca.add_routed = do_routed ? 1 : 0;
  return launch_combine(h, ca, T, d, s0, pdl);
}

moe_status moe_forward_fp8(moe_handle h, const void* x, int64_t T, const moe_router* router,
                           const moe_experts_fp8* experts, const moe_experts_fp8* shared, int32_t K, void* out,
                           void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  const moe_config& c = h->cfg;
  if (!(c.flags & MOE_FLAG_FP8)) return MOE_ERR_UNSUPPORTED;
  h->last_forward = 0;  // the workspace will hold FP8 rows: no backward follows
  if (T < 0 || T > c.max_tokens) return MOE_ERR_SHAPE;
  if (K < 1 || K > c.max_k || K > c.n_routed) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!router || !experts) return MOE_ERR_INVALID_ARG;
  if ((c.n_shared > 0) != (shared != nullptr)) return MOE_ERR_INVALID_ARG;
  auto complete = [](const moe_experts_fp8* e) {
    return e->w_gate && e->w_up && e->w_down && e->s_gate && e->s_up && e->s_down;
  };
  if (!x || !out || !router->weight || !complete(experts) || (shared && !complete(shared))) return MOE_ERR_INVALID_ARG;
  const bool sigmoid = c.gate == MOE_GATE_SIGMOID_BIASED;
  if (sigmoid ? router->logit_bias != nullptr : router->select_bias != nullptr) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, out, router->weight, router->logit_bias, router->select_bias, experts->w_gate,
                        experts->w_up, experts->w_down, shared ? shared->w_gate : nullptr,
                        shared ? shared->w_up : nullptr, shared ? shared->w_down : nullptr};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_ALIGNMENT;
  const int64_t d = c.d_model, N = c.n_routed, I = c.d_ff, Ks = c.n_shared, Is = c.d_ff_shared;
  const size_t out_bytes = size_t(T) * d * 2;
  const size_t wsz = size_t(N) * I * d, swsz = size_t(Ks) * Is * d;
  if (overlaps(out, out_bytes, x, out_bytes) || overlaps(out, out_bytes, router->weight, size_t(N) * d * 2) ||
      overlaps(out, out_bytes, experts->w_gate, wsz) || overlaps(out, out_bytes, experts->w_up, wsz) ||
      overlaps(out, out_bytes, experts->w_down, wsz) ||
      (shared && (overlaps(out, out_bytes, shared->w_gate, swsz) || overlaps(out, out_bytes, shared->w_up, swsz) ||
                  overlaps(out, out_bytes, shared->w_down, swsz))))
    return MOE_ERR_INVALID_ARG;

  DeviceGuard guard(h->device);
  cudaStream_t s0 = static_cast<cudaStream_t>(stream);
  const Layout& L = h->L;
  const bool do_shared = Ks > 0 && !(c.flags & MOE_FLAG_NO_SHARED);
  const bool do_routed = !(c.flags & MOE_FLAG_NO_ROUTED);
  // FP8 weight codes: W_gate / W_up [n][I][d] and W_down [n][d][I], 128-byte rows of K, 128-row boxes
  // (W_down 256: one box holds a tile's 256 output rows)
  bool ok = refresh_u8(h->tm8_wg, experts->w_gate, N, I, d, kF8BoxRowsW, 3) &&
            refresh_u8(h->tm8_wu, experts->w_up, N, I, d, kF8BoxRowsW, 3) &&
            refresh_u8(h->tm8_wd, experts->w_down, N, d, I, kF8BoxRowsWd, 3);
  if (shared)
    ok = ok && refresh_u8(h->tm8_swg, shared->w_gate, 1, Ks * Is, d, kF8BoxRowsW, 3) &&
         refresh_u8(h->tm8_swu, shared->w_up, 1, Ks * Is, d, kF8BoxRowsW, 3) &&
         refresh_u8(h->tm8_swd, shared->w_down, Ks, d, Is, kF8BoxRowsWd, 3);
  if (!ok) return MOE_ERR_CUDA;
  const bool pdl = T <= kPdlMaxT;
  const int nblk = ceil_div(T, 128);

  RouterArgs ra;
  {
    const moe_status st = enqueue_router(h, x, T, router, K, s0, pdl, ra);
    if (st != MOE_OK) return st;
  }
  PermuteQuantArgs pq{};
  pq.p = permute_args(h, x, T, K, ra, do_routed);
  pq.xq_perm = h->at<uint8_t>(L.xq_perm);
  pq.xs_perm = h->at<uint8_t>(L.xs_perm);
  pq.xq = do_shared ? h->at<uint8_t>(L.xq) : nullptr;
  pq.xs = do_shared ? h->at<uint8_t>(L.xs) : nullptr;
  {
    KernelTimer kt(h, MOE_KERNEL_PERMUTE, s0);
    if (launch_pdl(permute_quant_kernel, dim3(nblk, pq.p.split), dim3(kPermThreads), 0, s0, 1, pdl, pq) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }

  // a decode batch: both expert GEMMs in one weight-streaming launch (decode_ffn8.cuh)
  const bool decode = T <= kDecodeMaxT && decode_token_blocks(T, K, N) <= kFfnMaxBlocks;
  if (decode && (do_routed || do_shared)) {
    const int64_t SI = Ks * Is;
    ok = refresh_u8(h->tm8_wd128, experts->w_down, N, d, I, kFfnBoxRowsW, 3);
    if (shared) ok = ok && refresh_u8(h->tm8_swd128, shared->w_down, Ks, d, Is, kFfnBoxRowsW, 3);
    if (!ok) return MOE_ERR_CUDA;
    Ffn8Args f8{};
    FfnArgs& f = f8.f;
    f.T = (int)T;
    f.kb_gu = (int)(d / kF8BK);
    if (do_routed) {
      f.G = (int)N;
      f.n_wb_gu = (int)(I / kFfnWB);
      f.n_wb_dn = (int)(d / kFfnWB);
      f.kb_dn = (int)(I / kF8BK);
      f.counts = ra.counts;
      f.row_start = ra.row_start;
      f.row_scale = h->at<float>(L.gate_perm);
      f.y = h->at<__nv_bfloat16>(L.y);
    }
    if (do_shared) {
      f.sh_blocks = ceil_div(T, kFfnTB);
      f.sh_n_wb_gu = (int)(SI / kFfnWB);
      f.sh_n_wb_dn = (int)(d / kFfnWB);
      f.sh_J = (int)Ks;
      f.sh_kb_per_j = (int)(Is / kF8BK);
      f.sh_k_per_j = (int)Is;
      f.ys = h->at<__nv_bfloat16>(L.ys);
    }
    f.I = (int)I;
    f.sh_cols = (int)SI;
    f.d = (int)d;
    f.ctr = h->at<uint32_t>(L.ffn_ctr);
    f.err = h->at<uint32_t>(L.err);
    f.timeout_ns = kTimeoutNs;
    f.debug_wait = (c.flags & MOE_FLAG_DEBUG_WAIT_TIMEOUT) ? 1 : 0;
    f8.x_atoms = h->at<uint8_t>(L.xs_perm);
    f8.xs_atoms = h->at<uint8_t>(L.xs);
    f8.hq = h->at<uint8_t>(L.hq);
    f8.h_atoms = h->at<uint8_t>(L.hs_perm);
    f8.hsq = h->at<uint8_t>(L.hsq);
    f8.hs_atoms = h->at<uint8_t>(L.hss);
    f8.s_gate = experts->s_gate;
    f8.s_up = experts->s_up;
    f8.s_down = experts->s_down;
    if (shared) {
      f8.sh_s_gate = shared->s_gate;
      f8.sh_s_up = shared->s_up;
      f8.sh_s_down = shared->s_down;
    }
    // an absent part's maps are never read; the present part's stand in
    const CUtensorMap& Wg = do_routed ? h->tm8_wg.map : h->tm8_swg.map;
    const CUtensorMap& Wu = do_routed ? h->tm8_wu.map : h->tm8_swu.map;
    const CUtensorMap& Wd = do_routed ? h->tm8_wd128.map : h->tm8_swd128.map;
    const CUtensorMap& Xr = do_routed ? h->tm_xq_perm32 : h->tm_xq32;
    const CUtensorMap& Hr = do_routed ? h->tm_hq32 : h->tm_hsq32;
    const CUtensorMap& Wsg = do_shared ? h->tm8_swg.map : h->tm8_wg.map;
    const CUtensorMap& Wsu = do_shared ? h->tm8_swu.map : h->tm8_wu.map;
    const CUtensorMap& Wsd = do_shared ? h->tm8_swd128.map : h->tm8_wd128.map;
    const CUtensorMap& Xs = do_shared ? h->tm_xq32 : h->tm_xq_perm32;
    const CUtensorMap& Hs = do_shared ? h->tm_hsq32 : h->tm_hq32;
    {
      KernelTimer kt(h, MOE_KERNEL_GATE_UP, s0);
      if (launch_pdl(decode_ffn8_kernel, dim3(h->num_sms), dim3(kFfnThreads), ffn8_smem_bytes(), s0, 1, pdl, Wg,
                     Wu, Xr, Wsg, Wsu, Xs, Wd, Hr, Wsd, Hs, f8) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
  }

  if (!decode && (do_routed || do_shared)) {
    const moe_status st = enqueue_fp8_expert_gemms(h, T, do_shared, do_routed ? (int)N : 0, ra.mtile128_start,
                                                   ra.row_start, experts, shared, s0, pdl);
    if (st != MOE_OK) return st;
  }

  CombineArgs ca{};
  ca.T = (int)T;
  ca.K = K;
  ca.d = (int)d;
  ca.x = static_cast<const __nv_bfloat16*>(x);
  ca.ys = do_shared ? h->at<__nv_bfloat16>(L.ys) : nullptr;
  ca.y = h->at<__nv_bfloat16>(L.y);
  ca.slot_of = h->at<int32_t>(L.slot);
  ca.out = static_cast<__nv_bfloat16*>(out);
  ca.add_residual = (c.flags & MOE_FLAG_NO_RESIDUAL) ? 0 : 1;
  ca.add_routed = do_routed ? 1 : 0;
  return launch_combine(h, ca, T, d, s0, pdl);
}

namespace {
moe_status forward_host_chunks(moe_handle h, const void* x_host, int64_t T, const moe_router* router,
                               const moe_experts* experts, const moe_shared* shared, int32_t K, void* out_host,
                               void* stream);
}  // namespace

moe_status moe_forward_host(moe_handle h, const void* x_host, int64_t T, const moe_router* router,
                            const moe_experts* experts, const moe_shared* shared, int32_t K, void* out_host,
                            void* stream) {
  const moe_status st = forward_host_chunks(h, x_host, T, router, experts, shared, K, out_host, stream);
  if (h) h->last_forward = 0;  // the workspace holds the device copies' (or the last chunk's) routing
  return st;
}

namespace {
moe_status forward_host_chunks(moe_handle h, const void* x_host, int64_t T, const moe_router* router,
                               const moe_experts* experts, const moe_shared* shared, int32_t K, void* out_host,
                               void* stream) {
  if (!h || !x_host || !out_host) return MOE_ERR_INVALID_ARG;
  if (h->cfg.ep_ranks > 1) return MOE_ERR_UNSUPPORTED;
  if (T < 0 || T > h->cfg.max_tokens) return MOE_ERR_SHAPE;
  if (T == 0) return MOE_OK;
  DeviceGuard guard(h->device);
  cudaStream_t s0 = static_cast<cudaStream_t>(stream);
  const size_t row_bytes = size_t(h->cfg.d_model) * 2;
  uint8_t* xd = h->ws + h->L.xdev;
  uint8_t* od = h->ws + h->L.outdev;
  const uint8_t* xh = static_cast<const uint8_t*>(x_host);
  uint8_t* oh = static_cast<uint8_t*>(out_host);
  // Tokens are independent, so a large batch runs in chunks: chunk c + 1 is
  // copied in and chunk c - 1 copied out on two copy streams while chunk c
  // computes on `stream` (16B prefill, T = 16384: the 67 MB copies each way
  // otherwise add their full time to the forward's).  The first and last
  // chunks are small (T/16) so that little copying is left exposed before the
  // first kernel and after the last; the middle chunks share the rest.
  const int middle = static_cast<int>(std::min<int64_t>(kHostChunks - 2, T / kHostChunkRows));
  if (middle <= 1) {
    if (cudaMemcpyAsync(xd, xh, size_t(T) * row_bytes, cudaMemcpyHostToDevice, s0) != cudaSuccess)
      return MOE_ERR_CUDA;
    const moe_status st = moe_forward(h, xd, T, router, experts, shared, K, od, stream);
    if (st != MOE_OK) return st;
    if (cudaMemcpyAsync(oh, od, size_t(T) * row_bytes, cudaMemcpyDeviceToHost, s0) != cudaSuccess)
      return MOE_ERR_CUDA;
    return cudaStreamSynchronize(s0) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  if (!h->host_ready) {
    bool ok = cudaStreamCreateWithFlags(&h->copy_in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&h->copy_out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&h->host_start, cudaEventDisableTiming) == cudaSuccess;
    for (int c = 0; c < kHostChunks && ok; ++c)
      ok = cudaEventCreateWithFlags(&h->in_done[c], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&h->fwd_done[c], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {  // release what was made, so that a later call starts over
      release_host_pipeline(h);
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    h->host_ready = true;
  }
  // finish everything in flight on all three streams before returning, also on an error
  auto finish = [&](moe_status st) {
    const bool ok = cudaStreamSynchronize(h->copy_in) == cudaSuccess &&
                    cudaStreamSynchronize(s0) == cudaSuccess && cudaStreamSynchronize(h->copy_out) == cudaSuccess;
    return st != MOE_OK ? st : ok ? MOE_OK : MOE_ERR_CUDA;
  };
  // the copies in start after the work already queued on `stream`
  if (cudaEventRecord(h->host_start, s0) != cudaSuccess ||
      cudaStreamWaitEvent(h->copy_in, h->host_start, 0) != cudaSuccess)
    return finish(MOE_ERR_CUDA);
  const int chunks = middle + 2;
  const int64_t edge = T / 16;
  auto rows_of = [&](int c) -> int64_t {  // first row of chunk c (c == chunks: T)
    if (c <= 0) return 0;
    if (c >= chunks) return T;
    if (c == chunks - 1) return T - edge;
    return edge + (T - 2 * edge) * (c - 1) / middle;
  };
  for (int c = 0; c < chunks; ++c) {
    const size_t off = size_t(rows_of(c)) * row_bytes, n = size_t(rows_of(c + 1) - rows_of(c)) * row_bytes;
    if (cudaMemcpyAsync(xd + off, xh + off, n, cudaMemcpyHostToDevice, h->copy_in) != cudaSuccess ||
        cudaEventRecord(h->in_done[c], h->copy_in) != cudaSuccess)
      return finish(MOE_ERR_CUDA);
  }
  for (int c = 0; c < chunks; ++c) {
    const size_t off = size_t(rows_of(c)) * row_bytes, n = size_t(rows_of(c + 1) - rows_of(c)) * row_bytes;
    if (cudaStreamWaitEvent(s0, h->in_done[c], 0) != cudaSuccess) return finish(MOE_ERR_CUDA);
    const moe_status st =
        moe_forward(h, xd + off, rows_of(c + 1) - rows_of(c), router, experts, shared, K, od + off, stream);
    if (st != MOE_OK) return finish(st);
    if (cudaEventRecord(h->fwd_done[c], s0) != cudaSuccess ||
        cudaStreamWaitEvent(h->copy_out, h->fwd_done[c], 0) != cudaSuccess ||
        cudaMemcpyAsync(oh + off, od + off, n, cudaMemcpyDeviceToHost, h->copy_out) != cudaSuccess)
      return finish(MOE_ERR_CUDA);
  }
  return finish(MOE_OK);
}
}  // namespace

// ---------------------------------------------------------------------------
// Expert parallelism: the four steps of a forward and the peers' workspaces
// ---------------------------------------------------------------------------

static_assert(sizeof(cudaIpcMemHandle_t) == 64, "the header promises 64-byte IPC handles");
static_assert(kEpRowAlign == kExpertRowAlign, "the owner's row buffer has the single-GPU layout");

moe_status moe_ep_workspace(moe_handle h, void** workspace) {
  if (!h || !workspace || h->cfg.ep_ranks < 2) return MOE_ERR_INVALID_ARG;
  *workspace = h->ws;
  return MOE_OK;
}

moe_status moe_ep_set_peers(moe_handle h, void* const* workspaces) {
  if (!h || !workspaces || h->cfg.ep_ranks < 2) return MOE_ERR_INVALID_ARG;
  const int G = h->cfg.ep_ranks;
  if (workspaces[h->cfg.ep_rank] != h->ws) return MOE_ERR_INVALID_ARG;
  for (int r = 0; r < G; ++r)
    if (!workspaces[r] || (reinterpret_cast<uintptr_t>(workspaces[r]) & 255u)) return MOE_ERR_INVALID_ARG;
  for (int r = 0; r < G; ++r) h->peers.ws[r] = static_cast<uint8_t*>(workspaces[r]);
  h->peers_set = true;
  return MOE_OK;
}

moe_status moe_ep_ipc_handle(moe_handle h, void* handle) {
  if (!h || !handle || h->cfg.ep_ranks < 2) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  cudaIpcMemHandle_t m;
  if (cudaIpcGetMemHandle(&m, h->ws) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  std::memcpy(handle, &m, sizeof(m));
  return MOE_OK;
}

namespace {
void close_ipc_peers(moe_ctx* h) {
  for (int r = 0; r < kEpMaxRanks; ++r) {
    if (h->ipc_opened[r]) cudaIpcCloseMemHandle(h->peers.ws[r]);
    h->ipc_opened[r] = false;
  }
  h->peers_set = false;
}
}  // namespace

moe_status moe_ep_open_peers(moe_handle h, const void* handles) {
  if (!h || !handles || h->cfg.ep_ranks < 2) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  close_ipc_peers(h);
  const int G = h->cfg.ep_ranks, me = h->cfg.ep_rank;
  for (int r = 0; r < G; ++r) {
    if (r == me) {
      h->peers.ws[r] = h->ws;
      continue;
    }
    cudaIpcMemHandle_t m;
    std::memcpy(&m, static_cast<const uint8_t*>(handles) + 64 * r, sizeof(m));
    void* p = nullptr;
    if (cudaIpcOpenMemHandle(&p, m, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
      cudaGetLastError();
      close_ipc_peers(h);
      return MOE_ERR_CUDA;
    }
    h->peers.ws[r] = static_cast<uint8_t*>(p);
    h->ipc_opened[r] = true;
  }
  h->peers_set = true;
  return MOE_OK;
}

moe_status moe_ep_route(moe_handle h, const void* x, int64_t T, const moe_router* router, int32_t K,
                        void* stream) {
  if (!h || h->cfg.ep_ranks < 2) return MOE_ERR_INVALID_ARG;
  const moe_config& c = h->cfg;
  if (T < 0 || T > c.max_tokens) return MOE_ERR_SHAPE;
  if (K < 1 || K > c.max_k || K > c.n_routed) return MOE_ERR_INVALID_ARG;
  if (!router || !router->weight || (T > 0 && !x)) return MOE_ERR_INVALID_ARG;
  const bool sigmoid = c.gate == MOE_GATE_SIGMOID_BIASED;
  if (sigmoid ? router->logit_bias != nullptr : router->select_bias != nullptr) return MOE_ERR_INVALID_ARG;
  for (const void* p : {x, router->weight, static_cast<const void*>(router->logit_bias),
                        static_cast<const void*>(router->select_bias)})
    if (p && !aligned16(p)) return MOE_ERR_ALIGNMENT;
  DeviceGuard guard(h->device);
  cudaStream_t s0 = static_cast<cudaStream_t>(stream);
  h->ep_stage = 0;
  h->ep_x = x;
  h->ep_T = T;
  h->ep_K = K;
  if (T == 0) {
    // no tokens: counts of zero for the other ranks' plans
    h->last_stream = s0;
    h->last_T = 0;
    h->last_K = K;
    if (cudaMemsetAsync(h->ws + h->L.counts, 0, size_t(c.n_routed) * 4, s0) != cudaSuccess) return MOE_ERR_CUDA;
  } else {
    RouterArgs ra;
    const moe_status st = enqueue_router(h, x, T, router, K, s0, false, ra, 0);
    if (st != MOE_OK) return st;
  }
  h->ep_stage = 1;
  return MOE_OK;
}

moe_status moe_ep_dispatch(moe_handle h, void* stream) {
  if (!h || h->cfg.ep_ranks < 2 || !h->peers_set || h->ep_stage != 1) return MOE_ERR_INVALID_ARG;
  const moe_config& c = h->cfg;
  const Layout& L = h->L;
  DeviceGuard guard(h->device);
  cudaStream_t s0 = static_cast<cudaStream_t>(stream);
  const int G = c.ep_ranks, N = c.n_routed;
  const int64_t T = h->ep_T;
  KernelTimer kt(h, MOE_KERNEL_PERMUTE, s0);
  EpPlanArgs pa{};
  pa.G = G;
  pa.N = N;
  pa.rank = c.ep_rank;
  pa.counts_off = L.counts;
  pa.peers = h->peers;
  pa.base = h->at<int32_t>(L.ep_base);
  pa.counts_loc = h->at<int32_t>(L.ep_counts);
  pa.row_start = h->at<int32_t>(L.ep_row_start);
  pa.mtile_start = h->at<int32_t>(L.ep_mtile);
  pa.mtile128_start = h->at<int32_t>(L.ep_mtile128);
  ep_plan_kernel<<<1, kEpPlanThreads, ep_plan_smem_bytes(G, N), s0>>>(pa);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  if (T > 0) {
    const int nblk = ceil_div(T, 128);
    const int split = std::max(1, std::min(nblk <= 4 ? 32 : 8, (4 * h->num_sms + nblk - 1) / nblk));
    EpDispatchArgs da{};
    da.T = (int)T;
    da.K = h->ep_K;
    da.N = N;
    da.d = c.d_model;
    da.split = split;
    da.per_rank = N / G;
    da.idx = h->at<int32_t>(L.idx);
    da.gate = h->at<float>(L.gate);
    da.block_base = h->at<int32_t>(L.bc);
    da.offsets = h->at<int32_t>(L.offsets);
    da.base = pa.base;
    da.src = h->at<int32_t>(L.src);
    da.slot_of = h->at<int32_t>(L.slot);
    da.x = static_cast<const __nv_bfloat16*>(h->ep_x);
    da.xperm_off = L.x_perm;
    da.gate_off = L.gate_perm;
    da.peers = h->peers;
    da.tile_ctr = h->at<int>(L.tile_ctr);
    if (c.flags & MOE_FLAG_FP8) {
      // the FP8 layer sends each row's E4M3 codes and scale cells; the dense codes of x stay here
      const bool dense = c.n_shared > 0 && !(c.flags & MOE_FLAG_NO_SHARED);
      da.xq_off = L.xq_perm;
      da.xs_off = L.xs_perm;
      da.xq = dense ? h->at<uint8_t>(L.xq) : nullptr;
      da.xs = dense ? h->at<uint8_t>(L.xs) : nullptr;
      ep_dispatch_kernel<true><<<dim3(nblk, split), kPermThreads, 0, s0>>>(da);
    } else {
      ep_dispatch_kernel<false><<<dim3(nblk, split), kPermThreads, 0, s0>>>(da);
    }
  } else if (cudaMemsetAsync(h->ws + L.tile_ctr, 0, 8, s0) != cudaSuccess) {
    return MOE_ERR_CUDA;
  }
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  h->ep_stage = 2;
  return MOE_OK;
}

moe_status moe_ep_experts(moe_handle h, const moe_experts* experts, const moe_shared* shared, void* stream) {
  if (!h || h->cfg.ep_ranks < 2 || !h->peers_set || h->ep_stage != 2) return MOE_ERR_INVALID_ARG;
  const moe_config& c = h->cfg;
  if (c.flags & MOE_FLAG_FP8) return MOE_ERR_UNSUPPORTED;  // the rows were sent as FP8 codes
  if (!experts || !experts->w_gate || !experts->w_up || !experts->w_down) return MOE_ERR_INVALID_ARG;
  if ((c.n_shared > 0) != (shared != nullptr)) return MOE_ERR_INVALID_ARG;
  if (shared && (!shared->w_gate || !shared->w_up || !shared->w_down)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {experts->w_gate, experts->w_up, experts->w_down, shared ? shared->w_gate : nullptr,
                        shared ? shared->w_up : nullptr, shared ? shared->w_down : nullptr};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_ALIGNMENT;
  const int64_t d = c.d_model, I = c.d_ff, Ks = c.n_shared, Is = c.d_ff_shared;
  const int per = c.n_routed / c.ep_ranks;
  const int64_t T = h->ep_T;
  DeviceGuard guard(h->device);
  cudaStream_t s0 = static_cast<cudaStream_t>(stream);
  const Layout& L = h->L;
  const bool do_shared = Ks > 0 && !(c.flags & MOE_FLAG_NO_SHARED) && T > 0;
  const bool do_routed = !(c.flags & MOE_FLAG_NO_ROUTED);
  bool ok = refresh(h->tm_wg, experts->w_gate, 0, per, I, d, kGuBoxRowsB, 3);
  ok = ok && refresh(h->tm_wu, experts->w_up, 0, per, I, d, kGuBoxRowsB, 3);
  ok = ok && refresh(h->tm_wd, experts->w_down, 0, per, d, I, kBoxRowsB, 3);
  if (shared) {
    ok = ok && refresh(h->tm_swg, shared->w_gate, 0, 1, Ks * Is, d, kGuBoxRowsB, 3);
    ok = ok && refresh(h->tm_swu, shared->w_up, 0, 1, Ks * Is, d, kGuBoxRowsB, 3);
    ok = ok && refresh(h->tm_swd, shared->w_down, 0, Ks, d, Is, kBoxRowsB, 3);
  }
  if (!ok) return MOE_ERR_CUDA;
  if (do_routed || do_shared) {
    ExpertTables et{};
    if (do_routed)
      et = ExpertTables{per, h->at<int32_t>(L.ep_mtile128), h->at<int32_t>(L.ep_mtile),
                        h->at<int32_t>(L.ep_row_start), h->at<float>(L.gate_perm)};
    const moe_status st = enqueue_expert_gemms(h, T, do_shared, et, h->at<int>(L.tile_ctr), s0, false);
    if (st != MOE_OK) return st;
  }
  h->ep_stage = 3;
  return MOE_OK;
}

moe_status moe_ep_experts_fp8(moe_handle h, const moe_experts_fp8* experts, const moe_experts_fp8* shared,
                              void* stream) {
  if (!h || h->cfg.ep_ranks < 2 || !h->peers_set || h->ep_stage != 2) return MOE_ERR_INVALID_ARG;
  const moe_config& c = h->cfg;
  if (!(c.flags & MOE_FLAG_FP8)) return MOE_ERR_UNSUPPORTED;
  auto complete = [](const moe_experts_fp8* e) {
    return e->w_gate && e->w_up && e->w_down && e->s_gate && e->s_up && e->s_down;
  };
  if (!experts || !complete(experts)) return MOE_ERR_INVALID_ARG;
  if ((c.n_shared > 0) != (shared != nullptr) || (shared && !complete(shared))) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {experts->w_gate, experts->w_up, experts->w_down, shared ? shared->w_gate : nullptr,
                        shared ? shared->w_up : nullptr, shared ? shared->w_down : nullptr};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_ALIGNMENT;
  const int64_t d = c.d_model, I = c.d_ff, Ks = c.n_shared, Is = c.d_ff_shared;
  const int per = c.n_routed / c.ep_ranks;
  const int64_t T = h->ep_T;
  DeviceGuard guard(h->device);
  cudaStream_t s0 = static_cast<cudaStream_t>(stream);
  const Layout& L = h->L;
  const bool do_shared = Ks > 0 && !(c.flags & MOE_FLAG_NO_SHARED) && T > 0;
  const bool do_routed = !(c.flags & MOE_FLAG_NO_ROUTED);
  bool ok = refresh_u8(h->tm8_wg, experts->w_gate, per, I, d, kF8BoxRowsW, 3) &&
            refresh_u8(h->tm8_wu, experts->w_up, per, I, d, kF8BoxRowsW, 3) &&
            refresh_u8(h->tm8_wd, experts->w_down, per, d, I, kF8BoxRowsWd, 3);
  if (shared)
    ok = ok && refresh_u8(h->tm8_swg, shared->w_gate, 1, Ks * Is, d, kF8BoxRowsW, 3) &&
         refresh_u8(h->tm8_swu, shared->w_up, 1, Ks * Is, d, kF8BoxRowsW, 3) &&
         refresh_u8(h->tm8_swd, shared->w_down, Ks, d, Is, kF8BoxRowsWd, 3);
  if (!ok) return MOE_ERR_CUDA;
  if (do_routed || do_shared) {
    const moe_status st = enqueue_fp8_expert_gemms(h, T, do_shared, do_routed ? per : 0,
                                                   h->at<int32_t>(L.ep_mtile128), h->at<int32_t>(L.ep_row_start),
                                                   experts, shared, s0, false);
    if (st != MOE_OK) return st;
  }
  h->ep_stage = 3;
  return MOE_OK;
}

moe_status moe_ep_combine(moe_handle h, void* out, void* stream) {
  if (!h || h->cfg.ep_ranks < 2 || !h->peers_set || h->ep_stage != 3) return MOE_ERR_INVALID_ARG;
  const moe_config& c = h->cfg;
  const int64_t T = h->ep_T, d = c.d_model;
  if (T > 0 && !out) return MOE_ERR_INVALID_ARG;
  if (out && !aligned16(out)) return MOE_ERR_ALIGNMENT;
  if (overlaps(out, size_t(T) * d * 2, h->ep_x, size_t(T) * d * 2)) return MOE_ERR_INVALID_ARG;
  h->ep_stage = 4;
  if (T == 0) return MOE_OK;
  DeviceGuard guard(h->device);
  cudaStream_t s0 = static_cast<cudaStream_t>(stream);
  const Layout& L = h->L;
  const bool do_shared = c.n_shared > 0 && !(c.flags & MOE_FLAG_NO_SHARED);
  EpCombineArgs ca{};
  ca.T = (int)T;
  ca.K = h->ep_K;
  ca.d = (int)d;
  ca.per_rank = c.n_routed / c.ep_ranks;
  ca.x = static_cast<const __nv_bfloat16*>(h->ep_x);
  ca.ys = do_shared ? h->at<__nv_bfloat16>(L.ys) : nullptr;
  ca.idx = h->at<int32_t>(L.idx);
  ca.slot_of = h->at<int32_t>(L.slot);
  ca.y_off = L.y;
  ca.peers = h->peers;
  ca.out = static_cast<__nv_bfloat16*>(out);
  ca.add_residual = (c.flags & MOE_FLAG_NO_RESIDUAL) ? 0 : 1;
  ca.add_routed = (c.flags & MOE_FLAG_NO_ROUTED) ? 0 : 1;
  // the split of combine_kernel: whole rows per warp once the batch fills the SMs, shorter chunks below
  const int64_t resident = int64_t(h->num_sms) * 64;
  int cols = (int)d;
  if (T < resident) {
    const int chunks = ceil_div(2 * resident, T);
    cols = ceil_div(ceil_div(d, chunks), 256) * 256;
  }
  const int64_t warps = T * ceil_div(d, cols);
  KernelTimer kt(h, MOE_KERNEL_COMBINE, s0);
  ep_combine_kernel<<<ceil_div(warps * 32, 256), 256, 0, s0>>>(ca, cols);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_ep_plan(const int32_t* counts_all, int32_t G, int32_t n_routed, int32_t rank, int32_t* base,
                       int32_t* counts_local, int32_t* row_start, int32_t* mtile_start, int32_t* mtile128_start) {
  if (!counts_all || !base || !counts_local || !row_start || !mtile_start || !mtile128_start)
    return MOE_ERR_INVALID_ARG;
  if (G < 2 || G > kEpMaxRanks || n_routed < 1 || n_routed > kMaxRouted || n_routed % G || rank < 0 || rank >= G)
    return MOE_ERR_INVALID_ARG;
  for (int64_t i = 0; i < int64_t(G) * n_routed; ++i)
    if (counts_all[i] < 0) return MOE_ERR_INVALID_ARG;
  const int32_t* rows[kEpMaxRanks];
  for (int r = 0; r < G; ++r) rows[r] = counts_all + int64_t(r) * n_routed;
  for (int e = 0; e < n_routed; ++e) base[e] = ep_dest_base(rows, G, n_routed, rank, e);
  const int per = n_routed / G;
  for (int l = 0; l <= per; ++l)
    ep_owner_entry(rows, G, n_routed, rank, l, counts_local + l, row_start + l, mtile_start + l, mtile128_start + l);
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// The backward pass for the input and the router (backward.cuh states the formulas)
// ---------------------------------------------------------------------------

namespace {
cudaError_t launch_transpose(const void* src, void* dst, int batch, int R, int C, int dst_ld, int col0,
                             cudaStream_t s) {
  TransposeArgs t{};
  t.src = static_cast<const __nv_bfloat16*>(src);
  t.dst = static_cast<__nv_bfloat16*>(dst);
  t.R = R;
  t.C = C;
  t.dst_ld = dst_ld;
  t.col0 = col0;
  t.src_bs = static_cast<long long>(R) * C;
  t.dst_bs = static_cast<long long>(C) * dst_ld;
  transpose_bf16_kernel<<<dim3(ceil_div(C, kTrCols), ceil_div(R, kTrRows), batch), 256, 0, s>>>(t);
  return cudaGetLastError();
}

// the backward's buffers and their fixed descriptors, on first use
moe_status ensure_backward_buffers(moe_ctx* h) {
  if (h->bws) return MOE_OK;
  const moe_config& c = h->cfg;
  const Layout& L = h->L;
  const BwdLayout B = make_bwd_layout(c, L);
  if (cudaMalloc(&h->bws, B.total) != cudaSuccess) {
    cudaGetLastError();
    h->bws = nullptr;
    return MOE_ERR_NOMEM;
  }
  const int64_t N = c.n_routed, I = c.d_ff, d = c.d_model, Ks = c.n_shared, Is = c.d_ff_shared;
  bool ok = encode_bf16(&h->tm_b_dhperm, h->ws + L.y, 1, L.P, d, kBoxRowsA, 2);
  // the weight gradients' operands: row-major [K = forward rows][MN], 64 K rows x 64 MN elements per box
  ok = ok && encode_bf16(&h->tm_w_dy, h->bws + B.dy, 1, L.P, d, 64, 2);
  ok = ok && encode_bf16(&h->tm_w_m, h->bws + B.mrows, 1, L.P, I, 64, 2);
  ok = ok && encode_bf16(&h->tm_w_dab, h->bws + B.dab, 1, L.P, 2 * I, 64, 2);
  ok = ok && encode_bf16(&h->tm_w_xperm, h->ws + L.x_perm, 1, L.P, d, 64, 2);
  ok = ok && encode_bf16(&h->tm_b_dzb, h->bws + B.dzb, 1, c.max_tokens, B.Npad, kBoxRowsA, 2);
  ok = ok && encode_bf16(&h->tm_b_wdT, h->bws + B.wdT, N, I, d, kBoxRowsB, 3);
  ok = ok && encode_bf16(&h->tm_b_dab, h->bws + B.dab, 1, L.P, 2 * I, kBoxRowsA, 2);
  ok = ok && encode_bf16(&h->tm_b_wguT, h->bws + B.wguT, N, d, 2 * I, kBoxRowsB, 3);
  if (Ks > 0) {
    ok = ok && encode_bf16(&h->tm_b_swdT, h->bws + B.swdT, 1, Ks * Is, d, kBoxRowsB, 3);
    ok = ok && encode_bf16(&h->tm_b_dabs, h->bws + B.dabs, 1, L.Tpad, Ks * 2 * Is, kBoxRowsA, 2);
    ok = ok && encode_bf16(&h->tm_b_swguT, h->bws + B.swguT, Ks, d, 2 * Is, kBoxRowsB, 3);
    ok = ok && encode_bf16(&h->tm_w_ms, h->bws + B.msrows, 1, L.Tpad, Ks * Is, 64, 2);
    ok = ok && encode_bf16(&h->tm_w_dabs, h->bws + B.dabs, 1, L.Tpad, Ks * 2 * Is, 64, 2);
  } else {
    h->tm_w_ms = h->tm_w_m;
    h->tm_w_dabs = h->tm_w_dab;
    h->tm_b_swdT = h->tm_b_wdT;
    h->tm_b_dabs = h->tm_b_dab;
    h->tm_b_swguT = h->tm_b_wguT;
  }
  if (!ok) {
    cudaFree(h->bws);
    h->bws = nullptr;
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
}  // namespace

moe_status moe_backward(moe_handle h, const void* x, int64_t T, const moe_router* router, const moe_experts* experts,
                        const moe_shared* shared, int32_t K, const void* dh, void* dx, float* d_router,
                        float* d_logit_bias, float* dgate, const moe_weight_grads* wgrad, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  const moe_config& c = h->cfg;
  if (c.ep_ranks > 1) return MOE_ERR_UNSUPPORTED;
  if (T < 0 || T > c.max_tokens) return MOE_ERR_SHAPE;
  if (K < 1 || K > c.max_k || K > c.n_routed) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (h->last_forward != 1 || T != h->last_T || K != h->last_K) return MOE_ERR_INVALID_ARG;
  if (!x || !dh || !dx || !router || !router->weight || !experts || !experts->w_gate || !experts->w_up ||
      !experts->w_down)
    return MOE_ERR_INVALID_ARG;
  if ((c.n_shared > 0) != (shared != nullptr)) return MOE_ERR_INVALID_ARG;
  if (shared && (!shared->w_gate || !shared->w_up || !shared->w_down)) return MOE_ERR_INVALID_ARG;
  const bool sigmoid = c.gate == MOE_GATE_SIGMOID_BIASED;
  if (sigmoid ? router->logit_bias != nullptr : router->select_bias != nullptr) return MOE_ERR_INVALID_ARG;
  if (d_logit_bias && !router->logit_bias) return MOE_ERR_INVALID_ARG;  // no logit bias, no gradient of it
  if (wgrad && (!wgrad->w_gate || !wgrad->w_up || !wgrad->w_down ||
                (c.n_shared > 0 && (!wgrad->ws_gate || !wgrad->ws_up || !wgrad->ws_down))))
    return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, dh, dx, router->weight, experts->w_gate, experts->w_up, experts->w_down,
                        shared ? shared->w_gate : nullptr, shared ? shared->w_up : nullptr,
                        shared ? shared->w_down : nullptr, d_router, d_logit_bias, dgate,
                        wgrad ? wgrad->w_gate : nullptr, wgrad ? wgrad->w_up : nullptr,
                        wgrad ? wgrad->w_down : nullptr, wgrad ? wgrad->ws_gate : nullptr,
                        wgrad ? wgrad->ws_up : nullptr, wgrad ? wgrad->ws_down : nullptr};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_ALIGNMENT;
  const int64_t d = c.d_model, N = c.n_routed, I = c.d_ff, Ks = c.n_shared, Is = c.d_ff_shared;
  const size_t rows_bytes = size_t(T) * d * 2;
  if (overlaps(dx, rows_bytes, x, rows_bytes) || overlaps(dx, rows_bytes, dh, rows_bytes)) return MOE_ERR_INVALID_ARG;

  DeviceGuard guard(h->device);
  moe_status st = ensure_backward_buffers(h);
  if (st != MOE_OK) return st;
  cudaStream_t s0 = static_cast<cudaStream_t>(stream);
  const Layout& L = h->L;
  const BwdLayout B = make_bwd_layout(c, L);
  const bool do_shared = Ks > 0 && !(c.flags & MOE_FLAG_NO_SHARED);
  const bool do_routed = !(c.flags & MOE_FLAG_NO_ROUTED);
  const bool residual = !(c.flags & MOE_FLAG_NO_RESIDUAL);
  auto bw = [&](size_t off) { return h->bws + off; };
  h->last_stream = s0;
  // a GEMM in the per-group mode of down_gemm_kernel (fp32 out, rows >= split into out2; mn: bit 0 A and
  // bit 1 B MN-major, read through 64 x 64 boxes)
  auto kg_gemm = [&](const CUtensorMap& A, const CUtensorMap& Bm, int groups, const int32_t* kstart,
                     const int32_t* kcount, int M, int a_step, int bz_step, int split, int Ncols, int ld, float* out,
                     float* out2, int mn = 0, int b_col_step = 0) {
    GemmArgs k{};
    k.kg_groups = groups;
    k.kg_k_start = kstart;
    k.kg_k_count = kcount;
    k.kg_M = M;
    k.kg_m_tiles = ceil_div(M, kGemmBM);
    k.kg_a_row_step = a_step;
    k.kg_bz_step = bz_step;
    k.kg_split = split;
    k.kg_ld = ld;
    k.kg_mn = mn;
    k.kg_b_col_step = b_col_step;
    k.kg_out = out;
    k.kg_out2 = out2;
    k.n_tiles = ceil_div(Ncols, kGemmBN);
    k.n_limit = Ncols;
    k.err = h->at<uint32_t>(L.err);
    k.timeout_ns = kTimeoutNs;
    const int tiles = groups * k.kg_m_tiles * k.n_tiles;
    return launch_down(std::min(h->max_pairs, tiles), s0, false, A, Bm, A, Bm, k);
  };

  // descriptors of the caller's pointers
  bool ok = refresh(h->tm_x, x, T, 1, T, d, kGuBoxRowsA, 2);
  ok = ok && refresh(h->tm_b_dh, dh, T, 1, T, d, kBoxRowsA, 2);
  ok = ok && refresh(h->tm_wg, experts->w_gate, 0, N, I, d, kGuBoxRowsB, 3);
  ok = ok && refresh(h->tm_wu, experts->w_up, 0, N, I, d, kGuBoxRowsB, 3);
  if (shared) {
    ok = ok && refresh(h->tm_swg, shared->w_gate, 0, 1, Ks * Is, d, kGuBoxRowsB, 3);
    ok = ok && refresh(h->tm_swu, shared->w_up, 0, 1, Ks * Is, d, kGuBoxRowsB, 3);
  }
  if (!ok) return MOE_ERR_CUDA;

  // ---- K-major copies of the weights the data-gradient GEMMs contract over their other dimension ----
  cudaError_t e = cudaSuccess;
  if (do_routed) {
    e = launch_transpose(experts->w_down, bw(B.wdT), (int)N, (int)d, (int)I, (int)d, 0, s0);  // [N][I][d]
    if (e == cudaSuccess) e = launch_transpose(experts->w_gate, bw(B.wguT), (int)N, (int)I, (int)d, (int)(2 * I), 0, s0);
    if (e == cudaSuccess)
      e = launch_transpose(experts->w_up, bw(B.wguT), (int)N, (int)I, (int)d, (int)(2 * I), (int)I, s0);
  }
  if (do_shared && e == cudaSuccess) {
    e = launch_transpose(shared->w_down, bw(B.swdT), (int)Ks, (int)d, (int)Is, (int)d, 0, s0);  // [Ks Is][d]
    if (e == cudaSuccess)
      e = launch_transpose(shared->w_gate, bw(B.swguT), (int)Ks, (int)Is, (int)d, (int)(2 * Is), 0, s0);
    if (e == cudaSuccess)
      e = launch_transpose(shared->w_up, bw(B.swguT), (int)Ks, (int)Is, (int)d, (int)(2 * Is), (int)Is, s0);
  }
  if (e != cudaSuccess) return MOE_ERR_CUDA;

  const int32_t* slot_of = h->at<int32_t>(L.slot);
  const int TK = (int)(T * K);
  // ---- dm: routed rows (dh gathered into the expert order, times W_down) and shared rows ----
  if (do_routed) {
    // dy = g dh per routed row for the weight gradients
    __nv_bfloat16* dy = wgrad ? reinterpret_cast<__nv_bfloat16*>(bw(B.dy)) : nullptr;
    bwd_gather_kernel<<<ceil_div(int64_t(TK) * 32, 256), 256, 0, s0>>>(static_cast<const __nv_bfloat16*>(dh), slot_of,
                                                                       TK, K, (int)d, h->at<__nv_bfloat16>(L.y),
                                                                       h->at<float>(L.gate), dy);
    // the padding rows the weight-gradient GEMMs' K blocks reach, in X_perm and dy, as zeros (they may
    // hold an earlier call's rows)
    if (dy)
      zero_tail_rows_kernel<<<(int)N, 256, 0, s0>>>(h->at<int32_t>(L.row_start), h->at<int32_t>(L.counts), (int)d,
                                                     h->at<__nv_bfloat16>(L.x_perm), dy);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    GemmArgs g{};
    g.num_groups = (int)N;
    g.mtile_start = h->at<int32_t>(L.mtile);
    g.row_start = h->at<int32_t>(L.row_start);
    g.num_kb = ceil_div(d, kGemmBK);
    g.row_scale = nullptr;
    g.out = h->at<__nv_bfloat16>(L.h);
    g.n_tiles = ceil_div(I, kGemmBN);
    g.n_limit = (int)I;
    g.ld_out = (int)I;
    g.err = h->at<uint32_t>(L.err);
    g.timeout_ns = kTimeoutNs;
    if (launch_down(h->max_pairs, s0, false, h->tm_b_dhperm, h->tm_b_wdT, h->tm_b_dhperm, h->tm_b_wdT, g) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (do_shared && wgrad) {
    // the shared experts' weight gradients sum over the T tokens (dh and x read MN-major in place: the
    // maps end at T, so the rows past it read as zeros)
    if (!refresh(h->tm_w_dh, dh, T, 1, T, d, 64, 2) || !refresh(h->tm_w_x, x, T, 1, T, d, 64, 2))
      return MOE_ERR_CUDA;
    fill_dense_groups_kernel<<<1, 64, 0, s0>>>(reinterpret_cast<int32_t*>(bw(B.sh_kstart)),
                                               reinterpret_cast<int32_t*>(bw(B.sh_kcount)), (int)Ks, (int)T);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (do_shared) {
    GemmArgs g{};
    g.sh_rows = (int)T;
    g.sh_num_kb = ceil_div(d, kGemmBK);
    g.sh_J = 1;
    g.sh_k_per_j = (int)d;
    g.sh_out = h->at<__nv_bfloat16>(L.hs);
    g.n_tiles = ceil_div(Ks * Is, kGemmBN);
    g.n_limit = (int)(Ks * Is);
    g.ld_out = (int)(Ks * Is);
    g.err = h->at<uint32_t>(L.err);
    g.timeout_ns = kTimeoutNs;
    const int tiles = ceil_div(T, kGemmBM) * g.n_tiles;
    if (launch_down(std::min(h->max_pairs, tiles), s0, false, h->tm_b_dh.map, h->tm_b_swdT, h->tm_b_dh.map, h->tm_b_swdT, g) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
  }
  // ---- the recompute of a, b with the SwiGLU backward in its epilogue ----
  if (do_routed || do_shared) {
    if (cudaMemsetAsync(h->ws + L.tile_ctr, 0, 8, s0) != cudaSuccess) return MOE_ERR_CUDA;
    GateUpArgs g{};
    if (do_routed) {
      g.num_groups = (int)N;
      g.mtile_start = h->at<int32_t>(L.mtile128);
      g.row_start = h->at<int32_t>(L.row_start);
      g.n_tiles = ceil_div(I, kGuBN / 2);
      g.n_limit = (int)I;
      g.out = reinterpret_cast<__nv_bfloat16*>(bw(B.dab));
      g.ld_out = (int)(2 * I);
      g.dm = h->at<__nv_bfloat16>(L.h);
      g.ld_dm = (int)I;
      g.row_gate = h->at<float>(L.gate_perm);
      g.dg_part = reinterpret_cast<float*>(bw(B.dg_part));
      if (wgrad) {
        g.counts = h->at<int32_t>(L.counts);
        g.m_out = reinterpret_cast<__nv_bfloat16*>(bw(B.mrows));
      }
    }
    if (do_shared) {
      g.sh_rows = (int)T;
      g.sh_n_tiles = ceil_div(Ks * Is, kGuBN / 2);
      g.sh_n_limit = (int)(Ks * Is);
      g.sh_out = reinterpret_cast<__nv_bfloat16*>(bw(B.dabs));
      g.sh_ld_out = (int)(Ks * 2 * Is);
      g.sh_dm = h->at<__nv_bfloat16>(L.hs);
      g.sh_ld_dm = (int)(Ks * Is);
      g.sh_I = (int)Is;
      if (wgrad) g.sh_m_out = reinterpret_cast<__nv_bfloat16*>(bw(B.msrows));
    }
    g.num_kb = ceil_div(d, kGuBK);
    g.tile_ctr = h->at<int>(L.tile_ctr);
    g.die_split = h->num_sms / 2;
    g.err = h->at<uint32_t>(L.err);
    g.timeout_ns = kTimeoutNs;
    g.debug_wait = (c.flags & MOE_FLAG_DEBUG_WAIT_TIMEOUT) ? 1 : 0;
    const int sh_tiles = do_shared ? ceil_div(T, kGuBM) * g.sh_n_tiles : 0;
    const int ctas = do_routed || sh_tiles > h->num_sms ? h->num_sms : sh_tiles;
    const CUtensorMap& sA = do_shared ? h->tm_x.map : h->tm_xperm;
    const CUtensorMap& sG = do_shared ? h->tm_swg.map : h->tm_wg.map;
    const CUtensorMap& sU = do_shared ? h->tm_swu.map : h->tm_wu.map;
    if (launch_gateup(ctas, s0, false, h->tm_xperm, h->tm_wg.map, h->tm_wu.map, sA, sG, sU, g, true) != cudaSuccess)
      return MOE_ERR_CUDA;
    // ---- dx rows: [da | db] times [W_gate ; W_up] (routed rows into Y's buffer, shared into Ys') ----
    GemmArgs g2{};
    if (do_routed) {
      g2.num_groups = (int)N;
      g2.mtile_start = h->at<int32_t>(L.mtile);
      g2.row_start = h->at<int32_t>(L.row_start);
      g2.num_kb = ceil_div(2 * I, kGemmBK);
      g2.row_scale = nullptr;
      g2.out = h->at<__nv_bfloat16>(L.y);
    }
    if (do_shared) {
      g2.sh_rows = (int)T;
      g2.sh_num_kb = ceil_div(2 * Is, kGemmBK);
      g2.sh_J = (int)Ks;
      g2.sh_k_per_j = (int)(2 * Is);
      g2.sh_out = h->at<__nv_bfloat16>(L.ys);
    }
    g2.n_tiles = ceil_div(d, kGemmBN);
    g2.n_limit = (int)d;
    g2.ld_out = (int)d;
    g2.err = h->at<uint32_t>(L.err);
    g2.timeout_ns = kTimeoutNs;
    const int sh_tiles2 = do_shared ? ceil_div(T, kGemmBM) * g2.n_tiles : 0;
    const int pairs = do_routed || sh_tiles2 > h->max_pairs ? h->max_pairs : sh_tiles2;
    const CUtensorMap& sA2 = do_shared ? h->tm_b_dabs : h->tm_b_dab;
    const CUtensorMap& sB2 = do_shared ? h->tm_b_swguT : h->tm_b_wguT;
    if (launch_down(pairs, s0, false, h->tm_b_dab, h->tm_b_wguT, sA2, sB2, g2) != cudaSuccess) return MOE_ERR_CUDA;
  }
  // ---- the expert weights' gradients: per expert, sums over its rows (GEMMs with K = the rows) ----
  if (wgrad) {
    cudaError_t ke = cudaSuccess;
    if (do_routed) {
      const int32_t* ks = h->at<int32_t>(L.row_start);
      const int32_t* kc = h->at<int32_t>(L.counts);
      // MN-major operands straight from the row-major buffers: dW_down = dy^T m, dW_gate|up = [da|db]^T x
      ke = kg_gemm(h->tm_w_dy, h->tm_w_m, (int)N, ks, kc, (int)d, 0, 0, (int)d, (int)I, (int)I, wgrad->w_down,
                   nullptr, 3);
      if (ke == cudaSuccess)
        ke = kg_gemm(h->tm_w_dab, h->tm_w_xperm, (int)N, ks, kc, (int)(2 * I), 0, 0, (int)I, (int)d, (int)d,
                     wgrad->w_gate, wgrad->w_up, 3);
    } else {
      const size_t wb = size_t(N) * I * d * 4;
      if (cudaMemsetAsync(wgrad->w_gate, 0, wb, s0) != cudaSuccess ||
          cudaMemsetAsync(wgrad->w_up, 0, wb, s0) != cudaSuccess ||
          cudaMemsetAsync(wgrad->w_down, 0, wb, s0) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    if (Ks > 0 && do_shared && ke == cudaSuccess) {
      const int32_t* ks = reinterpret_cast<const int32_t*>(bw(B.sh_kstart));
      const int32_t* kc = reinterpret_cast<const int32_t*>(bw(B.sh_kcount));
      ke = kg_gemm(h->tm_w_dh.map, h->tm_w_ms, (int)Ks, ks, kc, (int)d, 0, 1, (int)d, (int)Is, (int)Is,
                   wgrad->ws_down, nullptr, 3, (int)Is);
      if (ke == cudaSuccess)
        ke = kg_gemm(h->tm_w_dabs, h->tm_w_x.map, (int)Ks, ks, kc, (int)(2 * Is), (int)(2 * Is), 0, (int)Is, (int)d,
                     (int)d, wgrad->ws_gate, wgrad->ws_up, 3);
    } else if (Ks > 0 && ke == cudaSuccess) {
      const size_t wb = size_t(Ks) * Is * d * 4;
      if (cudaMemsetAsync(wgrad->ws_gate, 0, wb, s0) != cudaSuccess ||
          cudaMemsetAsync(wgrad->ws_up, 0, wb, s0) != cudaSuccess ||
          cudaMemsetAsync(wgrad->ws_down, 0, wb, s0) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    if (ke != cudaSuccess) return MOE_ERR_CUDA;
  }
  // ---- the gates' gradient, and through them the router's ----
  float* dg = dgate ? dgate : reinterpret_cast<float*>(bw(B.dgate));
  float* dxr = nullptr;
  if (do_routed) {
    dg_reduce_kernel<<<ceil_div(TK, 256), 256, 0, s0>>>(reinterpret_cast<const float*>(bw(B.dg_part)), slot_of, TK,
                                                         ceil_div(I, kGuBN / 2), dg);
    // the router's three contractions on the tensor cores (the GEMM's per-group mode, one group
    // or a K split into segments): z = x E^T, dx_router = dz E, dE = dz^T x
    if (!refresh(h->tm_b_E, router->weight, 0, 1, N, d, kBoxRowsB, 3)) return MOE_ERR_CUDA;
    int32_t* ks = reinterpret_cast<int32_t*>(bw(B.rt_kstart));
    int32_t* kc = reinterpret_cast<int32_t*>(bw(B.rt_kcount));
    const int Np = (int)B.Npad;
    fill_segments_kernel<<<1, 32, 0, s0>>>(ks, kc, 1, (int)d, (int)d);
    if (kg_gemm(h->tm_x.map, h->tm_b_E.map, 1, ks, kc, (int)T, 0, 0, (int)T, (int)N, Np,
                reinterpret_cast<float*>(bw(B.zf)), nullptr) != cudaSuccess)
      return MOE_ERR_CUDA;
    RouterDzArgs rz{};
    rz.T = (int)T;
    rz.N = (int)N;
    rz.Npad = Np;
    rz.K = K;
    rz.sigmoid = sigmoid ? 1 : 0;
    rz.z = reinterpret_cast<const float*>(bw(B.zf));
    rz.logit_bias = router->logit_bias;
    rz.idx = h->at<int32_t>(L.idx);
    rz.dgate = dg;
    rz.dz = reinterpret_cast<float*>(bw(B.dz));
    rz.dzb = reinterpret_cast<__nv_bfloat16*>(bw(B.dzb));
    router_dz_kernel<<<ceil_div(T * 32, 256), 256, 0, s0>>>(rz);
    // dx_router = dz E: dz K-major, E [mN][d] read MN-major in place (its rows past mN read as zeros)
    if (!refresh(h->tm_w_E, router->weight, N, 1, N, d, 64, 2)) return MOE_ERR_CUDA;
    fill_segments_kernel<<<1, 32, 0, s0>>>(ks + 1, kc + 1, 1, (int)N, (int)N);
    dxr = reinterpret_cast<float*>(bw(B.dxr));
    if (kg_gemm(h->tm_b_dzb, h->tm_w_E.map, 1, ks + 1, kc + 1, (int)T, 0, 0, (int)T, (int)d, (int)d, dxr, nullptr,
                2) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (d_router) {
      // dE = dz^T x over token segments summed in segment order, both operands MN-major in place (the
      // maps end at T, so the rows past it read as zeros)
      if (!refresh(h->tm_w_dzb, bw(B.dzb), T, 1, T, Np, 64, 2) || !refresh(h->tm_w_x, x, T, 1, T, d, 64, 2))
        return MOE_ERR_CUDA;
      const int want = (int)std::max<int64_t>(1, std::min<int64_t>(kDeMaxSegments, T / 512));
      const int seg = ceil_div(ceil_div(T, want), 64) * 64;
      const int segs = ceil_div(T, seg);
      fill_segments_kernel<<<1, 32, 0, s0>>>(ks, kc, segs, seg, (int)T);
      float* part = reinterpret_cast<float*>(bw(B.de_part));
      if (kg_gemm(h->tm_w_dzb.map, h->tm_w_x.map, segs, ks, kc, (int)N, 0, 0, (int)N, (int)d, (int)d, part,
                  nullptr, 3) != cudaSuccess)
        return MOE_ERR_CUDA;
      router_de_reduce_kernel<<<ceil_div(N * d, 256), 256, 0, s0>>>(part, segs, size_t(N) * d, d_router);
    }
    if (d_logit_bias) column_sum_kernel<<<ceil_div(N, 256), 256, 0, s0>>>(rz.dz, (int)T, (int)N, d_logit_bias);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  } else {
    // the routed term left out: the gates and the router have no gradient
    if (dgate && cudaMemsetAsync(dgate, 0, size_t(TK) * 4, s0) != cudaSuccess) return MOE_ERR_CUDA;
    if (d_router && cudaMemsetAsync(d_router, 0, size_t(N) * d * 4, s0) != cudaSuccess) return MOE_ERR_CUDA;
    if (d_logit_bias && cudaMemsetAsync(d_logit_bias, 0, size_t(N) * 4, s0) != cudaSuccess) return MOE_ERR_CUDA;
  }
  // ---- dx = dh + shared rows + router term + the K routed rows (k ascending) ----
  BwdCombineArgs bc{};
  bc.T = (int)T;
  bc.K = K;
  bc.d = (int)d;
  bc.dh = residual ? static_cast<const __nv_bfloat16*>(dh) : nullptr;
  bc.dxs = do_shared ? h->at<__nv_bfloat16>(L.ys) : nullptr;
  bc.dx_router = dxr;
  bc.dx_perm = do_routed ? h->at<__nv_bfloat16>(L.y) : nullptr;
  bc.slot_of = slot_of;
  bc.dx = static_cast<__nv_bfloat16*>(dx);
  const int64_t resident = int64_t(h->num_sms) * 64;
  int cols = (int)d;
  if (T < resident) cols = ceil_div(ceil_div(d, ceil_div(2 * resident, T)), 256) * 256;
  const int64_t warps = T * ceil_div(d, cols);
  bwd_combine_kernel<<<ceil_div(warps * 32, 256), 256, 0, s0>>>(bc, cols);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_get_routing(moe_handle h, int32_t* idx, float* gate, int32_t* counts, int32_t* offsets,
                           int32_t* src, void* stream) {
  if (!h) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t tk = size_t(h->last_T) * h->last_K;
  const int64_t N = h->cfg.n_routed;
  const Layout& L = h->L;
  bool ok = true;
  auto cp = [&](void* dst, size_t off, size_t bytes) {
    if (dst && bytes) ok = ok && cudaMemcpyAsync(dst, h->ws + off, bytes, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
  };
  cp(idx, L.idx, tk * 4);
  cp(gate, L.gate, tk * 4);
  cp(counts, L.counts, N * 4);
  cp(offsets, L.offsets, (N + 1) * 4);
  cp(src, L.src, tk * 4);
  return ok ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_update_bias(moe_handle h, float* bias, float gamma, void* stream) {
  if (!h || !bias || (reinterpret_cast<uintptr_t>(bias) & 3u) || !std::isfinite(gamma)) return MOE_ERR_INVALID_ARG;
  if (h->last_T <= 0) return MOE_ERR_INVALID_ARG;  // no loads to balance yet
  DeviceGuard guard(h->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  bias_update_kernel<<<1, kBiasThreads, 0, s>>>(bias, h->at<int32_t>(h->L.counts), h->cfg.n_routed, gamma);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_status_query(moe_handle h) {
  if (!h) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (cudaStreamSynchronize(h->last_stream) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t err = 0;
  if (cudaMemcpy(&err, h->ws + h->L.err, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (err) {
    // a kernel that gave up may have left the decode FFN's counters part-counted
    if (cudaMemset(h->ws + h->L.err, 0, 4) != cudaSuccess ||
        cudaMemset(h->ws + h->L.ffn_ctr, 0, ffn_counter_bytes()) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_ERR_TIMEOUT;
  }
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_set_timing(moe_handle h, uint32_t kernel_mask) {
  if (!h || (kernel_mask & ~MOE_TIMING_ALL)) return MOE_ERR_INVALID_ARG;
  h->timing_mask = kernel_mask;
  return MOE_OK;
}

moe_status moe_kernel_times(moe_handle h, float* total_ms, int32_t* launches) {
  if (!h) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  moe_status st = MOE_OK;
  for (int k = 0; k < MOE_KERNEL_COUNT; ++k) {
    double sum = 0.0;
    const size_t used = h->ev_used[k];
    for (size_t i = 0; i + 1 < used; i += 2) {
      float ms = 0.f;
      if (cudaEventSynchronize(h->ev_pool[k][i + 1]) != cudaSuccess ||
          cudaEventElapsedTime(&ms, h->ev_pool[k][i], h->ev_pool[k][i + 1]) != cudaSuccess) {
        st = MOE_ERR_CUDA;
        break;
      }
      sum += ms;
    }
    if (total_ms) total_ms[k] = static_cast<float>(sum);
    if (launches) launches[k] = static_cast<int32_t>(used / 2);
    h->ev_used[k] = 0;
  }
  return st;
}

moe_status moe_destroy(moe_handle h) {
  if (!h) return MOE_OK;
  {
    DeviceGuard guard(h->device);
    cudaDeviceSynchronize();
    for (auto& pool : h->ev_pool)
      for (cudaEvent_t e : pool) cudaEventDestroy(e);
    release_host_pipeline(h);
    close_ipc_peers(h);
    if (h->bws) cudaFree(h->bws);
    if (h->ws) cudaFree(h->ws);
  }
  delete h;
  return MOE_OK;
}

}  // extern "C"
