// Decode entry point that allocates nothing: the split partials and per-(b, h)
// completion counters live in a file-scope device array instead of a caller
// workspace.  For callers that cannot call cudaMalloc (see wsvd.h).
#include <map>
#include <mutex>

#include "wsvd_internal.h"

namespace {

// Every GPU that loads the library holds this array until the process exits.
constexpr size_t kScratchBytes = (size_t)WSVD_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_mu;
std::map<int, void*> g_scratch_addr;  // device ordinal -> device address of g_decode_scratch

// Device address of the scratch array on the current device.  Host code only
// sees a host-side stand-in for the array's name, so the address is looked up
// once per device (that device current) and cached.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WSVD_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = g_scratch_addr.find(dev);
  if (it != g_scratch_addr.end()) {
    *out = it->second;
    return WSVD_OK;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return WSVD_ERR_CUDA;
  g_scratch_addr[dev] = p;
  *out = p;
  return WSVD_OK;
}

}  // namespace

extern "C" int wsvd_decode_attention_noalloc(int B, int H, int Hd, int r, int bits, int L_cap,
                                             const int32_t* seq_lens, const void* q, int q_dtype,
                                             const uint8_t* lat_k, const uint8_t* lat_v, const void* scale_k,
                                             const void* scale_v, const void* B_k, const void* B_v,
                                             float softmax_scale, float* out, int32_t* err, void* stream) {
  // The first checks of wsvd_decode_attention, in its order, before any CUDA
  // call; the rest of its validation runs with the scratch address below.
  if (B < 0 || H < 1 || L_cap < 0) return WSVD_ERR_INVALID_ARG;
  if (B == 0) return WSVD_OK;
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != WSVD_OK) return st;
  // A problem that needs more than the static array is refused as
  // WSVD_ERR_WORKSPACE_TOO_SMALL, like an undersized caller workspace.
  return wsvd::decode_with_scratch(B, H, Hd, r, bits, L_cap, seq_lens, q, q_dtype, lat_k, lat_v, scale_k, scale_v,
                                   B_k, B_v, softmax_scale, out, scratch, kScratchBytes, err,
                                   reinterpret_cast<cudaStream_t>(stream));
}
