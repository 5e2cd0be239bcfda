// qkn_decode_noalloc: the decode step for callers that cannot allocate GPU
// memory, with its scratch in a fixed array that lives in this library.
//
// Who needs it: code that is handed only input and output pointers and has no
// allocator of its own — an operator plugged into another engine's custom-op
// interface, a serving loop whose memory pool already owns all of HBM (where a
// stray cudaMalloc fails or fragments the pool), or a latency-critical loop
// that must not pay cudaMalloc's implicit synchronisation.  qkn_decode needs a
// caller-allocated workspace for its split-KV partial results; this entry
// point uses the static array below instead.
//
// The array is a file-scope __device__ object, so every GPU that loads the
// library holds QKN_NOALLOC_SCRATCH_BYTES of it until the process exits.  In
// host code its name is only a host-side stand-in, never a device address: the
// device address is looked up with cudaGetSymbolAddress, once per device, with
// that device current, on the first call made on that device.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

static __device__ __align__(256) unsigned char qkn_noalloc_scratch[QKN_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_on_device[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (nullptr on failure).
void* scratch_for_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_on_device[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, qkn_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    g_scratch_on_device[dev] = p;
  }
  return g_scratch_on_device[dev];
}

}  // namespace

extern "C" qkn_status qkn_decode_noalloc(const qkn_dims* dims, const qkn_cache* cache, qkn_ak_mode ak_mode,
                                         const void* q_tilde, const float* a_q, const void* q_rope_hat,
                                         const int32_t* block_table, int32_t max_blocks, const int32_t* seq_lens,
                                         int32_t batch, int32_t s_q, void* out, float* lse,
                                         int32_t* device_status, const qkn_decode_opts* opts, void* stream) {
  // Size check first, on the host, before anything is enqueued.
  size_t need = 0;
  qkn_status st = qkn_decode_workspace_size(dims, batch, s_q, 0, &need);
  if (st != QKN_OK) return st;
  if (need > (size_t)QKN_NOALLOC_SCRATCH_BYTES) return QKN_ERR_UNSUPPORTED;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (batch == 0) {
    // nothing to decode: the status the caller reads is QKN_OK (zero), written on the stream
    if (device_status && cudaMemsetAsync(device_status, 0, sizeof(int32_t), cs) != cudaSuccess) return QKN_ERR_CUDA;
    return QKN_OK;
  }

  void* scratch = scratch_for_current_device();
  if (!scratch) return QKN_ERR_CUDA;
  // The array keeps whatever the previous call left in it; only the status
  // word has to start from zero (everything else is written before it is read).
  if (cudaMemsetAsync(scratch, 0, qkn::kStatusBytes, cs) != cudaSuccess) return QKN_ERR_CUDA;
  st = qkn_decode(dims, cache, ak_mode, q_tilde, a_q, q_rope_hat, block_table, max_blocks, seq_lens, batch, s_q,
                  scratch, (size_t)QKN_NOALLOC_SCRATCH_BYTES, out, lse, opts, stream);
  if (st != QKN_OK) return st;
  if (device_status &&
      cudaMemcpyAsync(device_status, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, cs) != cudaSuccess)
    return QKN_ERR_CUDA;
  return QKN_OK;
}
