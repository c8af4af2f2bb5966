// bsa_static_ws.cu -- a forward entry point that needs no caller-supplied
// workspace and allocates nothing.
//
// Some callers cannot allocate device memory at the moment they run the
// attention forward: a plugin executed by an inference runtime whose
// contract forbids allocation inside its execute/enqueue step, or an engine
// that fixes its device-memory budget at start-up and must not grow it
// afterwards.  For them this entry point keeps its scratch in a fixed-size
// array that is part of the library image on every GPU that loads it.
//
// The scratch array below is a device symbol.  Host code must not use its
// name as an address: the host-side name is only a stand-in, and a kernel
// given it would fault or, where the GPU can reach host memory, silently
// use the wrong memory.  The device address is looked up once per device
// with cudaGetSymbolAddress and cached.  CUDA places the array on a device
// when this file's module is first used there, i.e. at that first lookup: the
// first call on each device grows device memory by the array's size, later
// calls allocate nothing.
#include <cuda_runtime.h>

#include <atomic>

#include "bsa_internal.h"

namespace {

// Largest forward workspace this entry point can serve (32 MiB).
constexpr size_t kStaticScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void *> g_scratch_addr[kMaxDevices];

// Device address of the scratch array on the current device (set-up on the
// first call per device; the lookup is idempotent, so a racing second
// lookup is harmless).
bsa_status scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSA_ERR_CUDA;
  void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
      return BSA_ERR_CUDA;
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return BSA_OK;
}

}  // namespace

extern "C" {

bsa_status bsa_fwd_static_workspace(const bsa_tensor *q, const bsa_tensor *k, const bsa_tensor *v,
                                    const bsa_tensor *index, const bsa_tensor *cu_seqlens_q,
                                    const bsa_tensor *cu_seqlens_kv,
                                    const bsa_tensor *seqused_kv, const bsa_tensor *block_table,
                                    const bsa_params *params, const bsa_tensor *out,
                                    const bsa_tensor *lse, void *stream) {
  size_t need = 0;
  bsa_status st = bsa_fwd_get_workspace(q, k, v, index, cu_seqlens_q, cu_seqlens_kv, seqused_kv,
                                        block_table, params, out, lse, &need);
  if (st == BSA_OK && need > kStaticScratchBytes) st = BSA_ERR_WORKSPACE;
  void *scratch = nullptr;
  if (st == BSA_OK) st = scratch_address(&scratch);
  if (st != BSA_OK) {
    bsa::drop_pending_events();  // a pair armed for this call ends with it
    return st;
  }
  return bsa_fwd(q, k, v, index, cu_seqlens_q, cu_seqlens_kv, seqused_kv, block_table, params, out,
                 lse, scratch, kStaticScratchBytes, stream);
}

}  // extern "C"
