// route_noalloc.cu -- routing (affinities, top-K, per-expert counts and
// offsets) for callers that cannot allocate device memory.
//
// Some callers own every byte of device memory up front: a serving runtime
// that plans a fixed memory budget before it starts, or a framework whose
// allocator must see every allocation.  Others sit in a latency-critical loop
// where cudaMalloc's implicit device-wide synchronisation is not acceptable.
// moe_create cannot serve them, because it allocates a workspace.  This entry
// point runs the same router kernel with its scratch (per-block expert
// histograms, the CTA completion counter, the padded expert starts) in a
// fixed file-scope device array instead, so it calls no cudaMalloc, cudaFree
// or allocating library routine.  The caller passes the inputs and outputs.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "../../include/fgs_moe.h"
#include "router_topk.cuh"

namespace {

// Largest batch the static scratch holds: 65536 tokens = 512 blocks of 128.
constexpr int64_t kNoAllocMaxTokens = 65536;
constexpr int kNoAllocMaxRouted = 256;
constexpr size_t kHeaderBytes = 4096;  // counter, error word, row and m-tile starts
constexpr size_t kScratchBytes =
    kHeaderBytes + static_cast<size_t>(kNoAllocMaxTokens / 128) * kNoAllocMaxRouted * sizeof(int32_t);
constexpr uint64_t kTimeoutNs = 2000ull * 1000 * 1000;
constexpr int kMaxDevices = 64;

// The scratch: 528 KB on every GPU that loads this library, held until the
// process exits.  In host code this name is only a host-side stand-in; the
// device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_route_scratch[kScratchBytes];

struct DeviceState {
  bool ready = false;
  uint8_t* scratch = nullptr;
};
DeviceState g_state[kMaxDevices];
std::mutex g_mutex;
PFN_cuTensorMapEncodeTiled_v12000 g_encode_fn = nullptr;

template <int K>
cudaError_t set_attrs_k(size_t smem) {
  cudaError_t e = cudaFuncSetAttribute(fgs::router_topk_kernel<K, true, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(fgs::router_topk_kernel<K, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(smem));
}

// Once per device, with that device current: the scratch's device address
// and the kernels' shared-memory limits.
moe_status setup_current_device(int dev, uint8_t** scratch) {
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& st = g_state[dev];
  if (!st.ready) {
    if (!g_encode_fn) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess)
        return MOE_ERR_CUDA;
      g_encode_fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    const size_t smem = fgs::router_smem_bytes(256);
    if (set_attrs_k<1>(smem) != cudaSuccess || set_attrs_k<2>(smem) != cudaSuccess ||
        set_attrs_k<3>(smem) != cudaSuccess || set_attrs_k<4>(smem) != cudaSuccess ||
        set_attrs_k<5>(smem) != cudaSuccess || set_attrs_k<6>(smem) != cudaSuccess ||
        set_attrs_k<7>(smem) != cudaSuccess || set_attrs_k<8>(smem) != cudaSuccess)
      return MOE_ERR_CUDA;
    st.scratch = static_cast<uint8_t*>(p);
    st.ready = true;
  }
  *scratch = st.scratch;
  return MOE_OK;
}

bool encode_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return g_encode_fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int K>
void launch_k(bool sigmoid, int grid, size_t smem, cudaStream_t s, const CUtensorMap& tx, const CUtensorMap& te,
              const fgs::RouterArgs& ra) {
  if (sigmoid)
    fgs::router_topk_kernel<K, true, false><<<grid, fgs::kRouterThreads, smem, s>>>(tx, te, ra);
  else
    fgs::router_topk_kernel<K, false, false><<<grid, fgs::kRouterThreads, smem, s>>>(tx, te, ra);
}

}  // namespace

extern "C" moe_status moe_route_noalloc(const void* x, int64_t T, int32_t d_model, const moe_router* router,
                                        int32_t n_routed, int32_t gate, int32_t K, int32_t* idx, float* gate_out,
                                        int32_t* counts, int32_t* offsets, uint32_t* err, void* stream) {
  if (T < 0 || T > kNoAllocMaxTokens) return MOE_ERR_SHAPE;
  if (n_routed < 1 || d_model < 16) return MOE_ERR_SHAPE;
  if (n_routed > kNoAllocMaxRouted || K > 8) return MOE_ERR_UNSUPPORTED;
  if (K < 1 || K > n_routed) return MOE_ERR_INVALID_ARG;
  if (gate != MOE_GATE_SOFTMAX && gate != MOE_GATE_SIGMOID_BIASED) return MOE_ERR_INVALID_ARG;
  if (d_model % 16) return MOE_ERR_ALIGNMENT;
  if (T == 0) return MOE_OK;
  if (!x || !router || !router->weight || !idx || !gate_out || !counts || !offsets || !err)
    return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(err) & 3u) return MOE_ERR_ALIGNMENT;
  const bool sigmoid = gate == MOE_GATE_SIGMOID_BIASED;
  if (sigmoid ? router->logit_bias != nullptr : router->select_bias != nullptr) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, router->weight, router->logit_bias, router->select_bias, idx, gate_out, counts, offsets};
  for (const void* p : ptrs)
    if (p && (reinterpret_cast<uintptr_t>(p) & 15u)) return MOE_ERR_ALIGNMENT;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  uint8_t* scratch = nullptr;
  const moe_status st = setup_current_device(dev, &scratch);
  if (st != MOE_OK) return st;

  const int N = n_routed;
  const int Npad = (N + 15) / 16 * 16;
  const int nblk = static_cast<int>((T + 127) / 128);
  CUtensorMap tx, te;
  if (!encode_2d(&tx, x, static_cast<uint64_t>(T), d_model, 128) ||
      !encode_2d(&te, router->weight, N, d_model, static_cast<uint32_t>(Npad)))
    return MOE_ERR_CUDA;

  // scratch layout: [0] CTA completion counter,
  // [256, +1028) row starts, [1536, +1028) and [2816, +1028) m-tile starts,
  // [4096, ...) block histograms
  uint32_t* done = reinterpret_cast<uint32_t*>(scratch);
  fgs::RouterArgs ra{};
  ra.T = static_cast<int>(T);
  ra.N = N;
  ra.Npad = Npad;
  ra.num_kb = (d_model + fgs::kBK - 1) / fgs::kBK;
  ra.nblk = nblk;
  ra.tmem_cols = Npad <= 32 ? 32u : Npad <= 64 ? 64u : Npad <= 128 ? 128u : 256u;
  ra.logit_bias = router->logit_bias;
  ra.select_bias = router->select_bias;
  ra.idx = idx;
  ra.gate = gate_out;
  ra.block_counts = reinterpret_cast<int32_t*>(scratch + kHeaderBytes);
  ra.counts = counts;
  ra.offsets = offsets;
  ra.row_start = reinterpret_cast<int32_t*>(scratch + 256);
  ra.mtile_start = reinterpret_cast<int32_t*>(scratch + 1536);
  ra.mtile128_start = reinterpret_cast<int32_t*>(scratch + 2816);
  ra.done_counter = done;
  ra.err = err;
  ra.timeout_ns = kTimeoutNs;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the counter must start at zero; the scratch keeps whatever the last call left
  if (cudaMemsetAsync(done, 0, sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  const size_t smem = fgs::router_smem_bytes(Npad);
  switch (K) {
    case 1: launch_k<1>(sigmoid, nblk, smem, s, tx, te, ra); break;
    case 2: launch_k<2>(sigmoid, nblk, smem, s, tx, te, ra); break;
    case 3: launch_k<3>(sigmoid, nblk, smem, s, tx, te, ra); break;
    case 4: launch_k<4>(sigmoid, nblk, smem, s, tx, te, ra); break;
    case 5: launch_k<5>(sigmoid, nblk, smem, s, tx, te, ra); break;
    case 6: launch_k<6>(sigmoid, nblk, smem, s, tx, te, ra); break;
    case 7: launch_k<7>(sigmoid, nblk, smem, s, tx, te, ra); break;
    default: launch_k<8>(sigmoid, nblk, smem, s, tx, te, ra); break;
  }
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
