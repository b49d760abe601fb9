// hs2_static.cu -- hs2_full_attn_select_static(): the full-attention +
// selection call with its scratch in a fixed, library-owned device array, for
// callers that are not allowed to allocate device memory themselves.
//
// Who needs it: code that only receives device pointers and a stream and may
// not call cudaMalloc -- for example a plugin inside a serving engine that
// has already reserved almost all HBM for its own KV-cache pool and forbids
// any further device allocation, or code whose calls are later recorded into
// a CUDA graph, where allocating is not permitted.  Such callers cannot hand
// hs2_full_attn_select() a workspace, so this entry point brings its own.
//
// The scratch is a file-scope __device__ array of kStaticScratchBytes (32 MiB);
// every GPU that loads the library holds it until the process exits.  Its
// device address is looked up once per device (cudaGetSymbolAddress, with
// that device current) on the first call made on that device.
#include <stdio.h>

#include <mutex>

#include "hs2.h"
#include "hs2_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

}  // namespace

extern "C" int hs2_full_attn_select_static(const hs2_heads *q, const hs2_cache *k_cache, const hs2_cache *v_cache,
                                           const int32_t *seq_lens, const int32_t *page_table, int32_t max_pages,
                                           int32_t window, int32_t k_global, hs2_heads *out, int32_t *idx_out,
                                           void *stream) {
  // The scratch need is the same as the workspace the allocating call needs.
  if (q && k_cache && k_cache->num_kv_heads > 0 && q->num_heads % k_cache->num_kv_heads == 0) {
    const int64_t t_cap = page_table ? (int64_t)max_pages * k_cache->page_size : (int64_t)k_cache->page_size;
    const size_t need = hs2_full_attn_select_workspace(q->batch, k_cache->num_kv_heads,
                                                       q->num_heads / k_cache->num_kv_heads, k_cache->head_dim, t_cap);
    if (need > kStaticScratchBytes) {
      char msg[256];
      snprintf(msg, sizeof msg,
               "this shape needs %zu bytes of scratch; the static scratch of hs2_full_attn_select_static holds %zu "
               "bytes (use hs2_full_attn_select with a caller workspace)",
               need, kStaticScratchBytes);
      return hs2::set_last_error(HS2_ERR_WORKSPACE, msg);
    }
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return hs2::set_last_error(HS2_ERR_CUDA, "no usable current CUDA device");
  void *scratch;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
      void *p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
      if (e != cudaSuccess || !p) {
        char msg[256];
        snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
        return hs2::set_last_error(HS2_ERR_CUDA, msg);
      }
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  return hs2_full_attn_select(q, k_cache, v_cache, seq_lens, page_table, max_pages, window, k_global, out, idx_out,
                              scratch, kStaticScratchBytes, stream);
}
