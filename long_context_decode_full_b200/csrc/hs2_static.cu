// hs2_static.cu -- hs2_full_attn_select_static(): the full-attention +
// selection call with its scratch in a fixed, library-owned device array, for
// callers that are not allowed to allocate device memory themselves.
//
// Who needs it: code that only receives device pointers and a stream and may
// not call cudaMalloc -- for example a plugin inside a serving engine that
// has reserved almost all HBM for its own KV-cache pool up front and forbids
// any later device allocation, or an extension of a runtime that plans every
// buffer before execution starts and hands its kernels no scratch.  Such
// callers cannot give hs2_full_attn_select() a workspace, so this entry point
// brings its own.
//
// The scratch is a file-scope __device__ array of kStaticScratchBytes (32 MiB);
// every GPU that loads the library holds it until the process exits.  In host
// code the array's name is only a stand-in, so its device address is looked
// up with cudaGetSymbolAddress once per CUDA context (with that context
// current), on the first call made in that context, and cached.  Word 0 of
// the array is the kernels' sticky error flag, which
// hs2_full_attn_select_static_status() reads and clears.
#include <stdio.h>

#include <mutex>

#include "hs2.h"
#include "hs2_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of the array in each CUDA context seen so far.  A module is
// loaded once per context, so the address is per context, not per device.
constexpr int kMaxContexts = 64;
struct CtxEntry {
  void *ctx;
  void *ptr;
};
CtxEntry g_entries[kMaxContexts];
int g_num_entries = 0;
std::mutex g_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// The array's device address in the current context (looked up on first use).
int scratch_address(void **out) {
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) return hs2::set_last_error(HS2_ERR_CUDA, "cuCtxGetCurrent is not available from the driver");
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return hs2::set_last_error(HS2_ERR_CUDA, "cuCtxGetCurrent failed");
  if (!ctx) {  // nothing bound yet: the symbol lookup binds the current device's primary context
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || get(&ctx) != CUDA_SUCCESS || !ctx)
      return hs2::set_last_error(HS2_ERR_CUDA, "no usable current CUDA device");
  }
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < g_num_entries; ++i)
    if (g_entries[i].ctx == ctx) {
      *out = g_entries[i].ptr;
      return HS2_OK;
    }
  if (g_num_entries == kMaxContexts)
    return hs2::set_last_error(HS2_ERR_CUDA, "more CUDA contexts than the static scratch keeps addresses for");
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
  if (e != cudaSuccess || !p) {
    char msg[256];
    snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
    return hs2::set_last_error(HS2_ERR_CUDA, msg);
  }
  g_entries[g_num_entries++] = CtxEntry{ctx, p};
  *out = p;
  return HS2_OK;
}

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
  void *scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc != HS2_OK) return rc;
  return hs2_full_attn_select(q, k_cache, v_cache, seq_lens, page_table, max_pages, window, k_global, out, idx_out,
                              scratch, kStaticScratchBytes, stream);
}

extern "C" int hs2_full_attn_select_static_status(void *stream) {
  void *scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc != HS2_OK) return rc;
  return hs2_workspace_status(scratch, kStaticScratchBytes, stream);
}

extern "C" int hs2_selftest_bounded_wait_static(void *stream) {
  void *scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc != HS2_OK) return rc;
  const cudaError_t e = hs2::launch_wait_selftest(static_cast<uint32_t *>(scratch), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof msg, "self-test launch: %s", cudaGetErrorString(e));
    return hs2::set_last_error(HS2_ERR_CUDA, msg);
  }
  return HS2_OK;
}
