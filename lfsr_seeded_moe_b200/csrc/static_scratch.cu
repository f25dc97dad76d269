// static_scratch.cu -- nslm_moe_seed_ffn_static: the decode expert FFN with its
// scratch memory built into the library instead of passed in by the caller.
//
// Who needs it: code that may not allocate device memory at call time.  A
// plug-in running inside a host application whose allocator owns the GPU's
// memory (a foreign cudaMalloc there fragments the pool or trips its leak
// accounting); a latency-critical loop where an allocation's implicit device
// synchronisation is not acceptable; a caller that is only handed input and
// output pointers and has no place to keep a workspace between calls.
//
// The scratch is a 1 MiB array in device memory that every GPU loading this
// library keeps until the process exits.  Host code cannot use the array's
// name as a device address (it denotes a host-side stand-in), so the device
// address is looked up once per device with cudaGetSymbolAddress, on the first
// call made while that device is current, and cached.
#include <mutex>

#include "common.cuh"
#include "moe.cuh"
#include "stackb.cuh"

namespace nslm {
namespace {

constexpr size_t kStaticScratchBytes = size_t(1) << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxScratchDevices = 64;
void *g_scratch_addr[kMaxScratchDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.
int32_t static_scratch_address(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_status(cudaErrorInvalidDevice);
  if (dev < 0 || dev >= kMaxScratchDevices) return NSLM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_status(e);
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return NSLM_OK;
}

}  // namespace

int32_t static_scratch_status_word(const int32_t **out) {
  void *p = nullptr;
  const int32_t st = static_scratch_address(&p);
  if (st == NSLM_OK) *out = static_cast<const int32_t *>(p);
  return st;
}

}  // namespace nslm

using namespace nslm;

extern "C" int32_t nslm_moe_seed_ffn_static(const nslm_seed_matrix *gate, const nslm_seed_matrix *up,
                                            const nslm_seed_matrix *down, int32_t E,
                                            const uint16_t *x_bf16, const int32_t *ids,
                                            const float *w, int32_t T, int32_t k, float *y,
                                            nslm_stream_t stream) {
  g_launches = 0;
  FfnDims d{};
  int32_t st = check_ffn_shapes(gate, up, down, E, d);
  if (st) return st;
  if (!x_bf16 || !ids || !w || !y) return NSLM_ERR_ARG;
  if (k < 1 || k > kMaxK || T < 0) return NSLM_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(y)) return NSLM_ERR_ALIGN;
  if (T == 0) return NSLM_OK;
  if (T > kMaxT) return NSLM_ERR_SHAPE;
  // the whole decode workspace must fit in the built-in array
  if (ffn_workspace(nullptr, T, k, d.hidden, d.inter, 1).bytes > kStaticScratchBytes)
    return NSLM_ERR_WORKSPACE;
  if ((st = check_device())) return st;
  void *scratch = nullptr;
  if ((st = static_scratch_address(&scratch))) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const FfnWorkspace fw = ffn_workspace(reinterpret_cast<char *>(scratch), T, k, d.hidden, d.inter, 1);
  // The routing kernel rewrites the plan and zeroes the down kernel's arrival
  // counters on every call, so whatever an earlier call left in the array is
  // harmless; h and the partial sums are written before they are read.
  if ((st = launch_route_plan(nullptr, ids, w, T, E, k, 1, fw.plans, nullptr, nullptr, fw.counters,
                              d.hidden, fw.sync, decode_slot_cap(d, T, k), nullptr, 0, s)))
    return st;
  int launches = 1;
  const nslm_moe_layer layer{*gate, *up, *down};
  st = launch_decode_stack(d, &layer, 1, x_bf16, T, k, fw, y, s, launches);
  if (st == NSLM_OK) g_launches = launches;
  return st;
}
