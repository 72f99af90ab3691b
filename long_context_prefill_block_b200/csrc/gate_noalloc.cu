// moba_gate_topk_noalloc: the gate/top-k call for callers that cannot
// allocate device memory.
//
// moba_gate_topk keeps its block means in a workspace the caller allocates.
// Some callers cannot do that: code that runs inside a host runtime which
// owns every byte of device memory and forbids cudaMalloc (inference
// engines with a fixed arena, plugin interfaces of other frameworks), and
// latency-critical paths where cudaMalloc's implicit device-wide
// synchronisation is not acceptable. This variant takes the block means'
// storage from a fixed array compiled into the library instead, so the
// caller passes only inputs and outputs.
//
// The array below is a file-scope __device__ object: every GPU that loads
// the library holds it until the process exits. In host code its name is
// only a host-side stand-in, not a device address, so the device address is
// looked up with cudaGetSymbolAddress once per device, with that device
// current, and cached. The status word (a __device__ symbol of api.cu) is
// reached the same way, so bad sequence offsets are reported as they are
// for moba_gate_topk; nothing here allocates.
#include <mutex>

#include "host_api.cuh"

namespace {

// Largest block-mean table this entry point accepts: 4 MiB of fp32, i.e.
// batch * ceil(max_seqlen / B) * Hkv * d <= 1,048,576 floats. The
// million-token GQA shape (B = 4096, 8 kv heads, d = 128) needs 262,144.
constexpr size_t kScratchBytes = size_t(4) << 20;

static __device__ __align__(256) float g_gate_scratch[kScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
float* g_scratch_ptr[kMaxDevices] = {};
int* g_status_ptr[kMaxDevices] = {};

// Device addresses of g_gate_scratch and of the status word on the current
// device; the first call on a device performs the lookups.
cudaError_t addresses_on_current_device(float** scratch, int** status) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_gate_scratch);
    if (e != cudaSuccess) return e;
    int* st = moba::status_word();
    if (!st) return cudaErrorInvalidSymbol;
    g_status_ptr[dev] = st;
    g_scratch_ptr[dev] = static_cast<float*>(ptr);
  }
  *scratch = g_scratch_ptr[dev];
  *status = g_status_ptr[dev];
  return cudaSuccess;
}

bool aligned32(const void* x) { return (reinterpret_cast<uintptr_t>(x) & 31) == 0; }

}  // namespace

extern "C" moba_status moba_gate_topk_noalloc(const moba_params* p, const void* q, const void* k,
                                              const int32_t* cu_seqlens, int32_t* idx,
                                              void* stream) {
  moba::Dims dm;
  const moba_status s = moba::validate(p, dm);
  if (s != MOBA_OK) return s;
  // the prefix-mean gate keeps T * Hq own-block scores: no room in the fixed
  // array; head-major k is a decode-cache layout, which no gate call takes
  if (dm.prefix || dm.kv_hm) return MOBA_ERR_UNSUPPORTED;
  if (dm.T == 0 || dm.batch == 0) return MOBA_OK;
  // the size limit is checked before the pointers, so that a refusal never
  // depends on what the pointers hold
  const size_t need = sizeof(float) * (size_t)dm.batch * dm.nb * dm.Hkv * dm.d;
  if (need > kScratchBytes) return MOBA_ERR_WORKSPACE;  // beyond the built-in 4 MiB
  if (!q || !k || !cu_seqlens || !idx || !aligned32(q) || !aligned32(k))
    return MOBA_ERR_INVALID_ARG;
  float* kbar = nullptr;
  int* status = nullptr;
  if (addresses_on_current_device(&kbar, &status) != cudaSuccess) return MOBA_ERR_CUDA;
  // Nothing has to start at zero: the mean-pool writes every slot of the
  // table that the gate reads (0 for blocks past a sequence's end).
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (moba::launch_meanpool(dm, k, cu_seqlens, kbar, status, st) != cudaSuccess)
    return MOBA_ERR_CUDA;
  if (moba::launch_gate(dm, q, kbar, nullptr, cu_seqlens, idx, status, st) != cudaSuccess)
    return MOBA_ERR_CUDA;
  return MOBA_OK;
}
