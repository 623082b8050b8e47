// vdn_branch_forward_static: the branch forward with its scratch in a fixed,
// library-owned device array instead of a caller-allocated workspace.
//
// For callers that cannot allocate device memory at the point where they run
// the branch: code that runs while a CUDA stream is being captured into a graph
// (cudaMalloc is not a stream operation and is refused during capture), and
// runtimes whose device memory is owned by a framework allocator or a fixed
// arena, with no cudaMalloc allowed on the inference path.  The caller still
// passes every input and the output.
#include <atomic>

#include "vdn.h"

namespace {

// Every GPU that loads this library holds this array until the process exits.
constexpr size_t kStaticWorkspaceBytes = size_t(64) << 20;   // 64 MiB
constexpr int kMaxDevices = 64;

// Host code must not take the address of this symbol directly: on the host it
// names a stand-in object, not device memory.  Its device address comes from
// cudaGetSymbolAddress, once per device.
__device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

std::atomic<void*> g_workspace_addr[kMaxDevices];

}  // namespace

extern "C" vdn_status vdn_branch_forward_static(const vdn_shape* shape, const void* q, const void* k, const void* v,
                                                const float* beta, const float* alpha, const void* gate,
                                                const float* rms_w, const float* conv_k_w, const float* conv_v_w,
                                                const float* text_state, int rule, float c, int chunk, int radius,
                                                void* out, void* stream) {
  // size check first: a problem whose scratch does not fit is refused before any CUDA call
  const size_t need = vdn_branch_workspace_size(shape, rule);
  if (need == 0) {
    // invalid shape or rule: let the regular validation name the error
    return vdn_branch_forward(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c,
                              chunk, radius, nullptr, 0, out, stream);
  }
  if (need > kStaticWorkspaceBytes) return VDN_ERR_WORKSPACE;

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return VDN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return VDN_ERR_UNSUPPORTED;
  void* ws = g_workspace_addr[dev].load(std::memory_order_acquire);
  if (!ws) {
    // set-up on the first call on this device (with the caller's device current)
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || !p) return VDN_ERR_CUDA;
    g_workspace_addr[dev].store(p, std::memory_order_release);
    ws = p;
  }
  // The forward clears the only workspace field that must start at zero (the
  // device status word) at the start of every call; all other scratch is fully
  // written before it is read.
  return vdn_branch_forward(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c, chunk,
                            radius, ws, kStaticWorkspaceBytes, out, stream);
}
