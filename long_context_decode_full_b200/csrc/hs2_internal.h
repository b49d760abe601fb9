// hs2_internal.h -- host-side launchers shared between the C-ABI layer and
// the kernel translation units (not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hs2_common.cuh"

namespace hs2 {

// Parameters of the full-attention (split over the context) kernels.
struct FullParams {
  const void *q;             // [B, Hq, D] (bf16, or f32 for the f32 path)
  const void *k, *v;         // caches (plain loads of the f32 path)
  const float *k_scale;      // E4M3 only
  const float *v_scale;
  const int32_t *seq_lens;   // [B]
  const int32_t *page_table; // [B, max_pages] or nullptr
  int32_t B, Hkv, G, D;
  int32_t page_size, max_pages;
  int64_t t_cap;             // logical capacity per sequence
  int64_t ustride;           // positions per unit in the workspace arrays (t_cap rounded up to 128)
  int64_t num_slots;
  int32_t N;                 // persistent CTAs (grid size)
  int32_t R;                 // record slots per unit
  int32_t tile;              // positions per tile
  int32_t kv_evict_first;    // K/V loads marked evict-first in L2 (when the logits fit in L2 beside them)
  float c;                   // 1/sqrt(D)
  FullWs ws;
};

struct ScoreParams {
  const int32_t *seq_lens;
  const int32_t *page_table;
  void *out;                 // [B, Hq, D] in out_dtype
  int32_t out_dtype;         // 0 f32, 1 bf16
  int32_t *idx_out;          // [B, Hkv, W + K]
  int32_t B, Hkv, G, D;
  int32_t page_size, max_pages;
  int64_t t_cap;
  int64_t ustride;
  int32_t window, k_global;
  int32_t N, R, tile;
  int32_t nsub;              // 512-position lists per unit: ceil(t_cap / 512)
  int32_t score_chunk;       // positions per score CTA (a power of two, 2048 .. 65536)
  int32_t filter_subs;       // 512-position sub-ranges per filter warp (1 or 2)
  int32_t ncomb;             // combine CTAs per unit (256 output elements each)
  float c;
  FullWs ws;
};

struct SparseParams {
  const void *q;             // [B, Hq, D]
  const void *k, *v;
  const float *k_scale, *v_scale;
  const int32_t *idx;        // [B, Hkv, L]
  void *out;                 // [B, Hq, D]
  int32_t B, Hkv, G, D;
  int32_t L;                 // idx_stride
  int32_t rows_per_cta;      // multiple of 16
  int32_t splits;            // CTAs per unit (cluster size)
  int32_t nbuf;              // gather buffers (one group each) per warp (1..4)
  int32_t warps;             // warps per CTA (4 or 8)
  int32_t nsl;               // 16-row slices per group (1 or 2)
  float c;
};

// Launch configuration chosen by the host for the tensor-core full kernel.
struct FullMmaConfig {
  int ncw;     // consumer warps
  int nstage;  // pipeline stages
  int nsl;     // 16-row slices per warp and tile (tile = 16 * ncw * nsl positions)
  int nt;      // 8-head MMA N-tiles per warp (1, or 2 for groups of 16 and more heads)
  int tc;      // 1: tcgen05 consumers (groups of 16 or 32 heads, d 128; ncw 4, nstage 3, nsl 2, nt 2)
};
// Shared memory of the tcgen05 attention kernel for a batch of B sequences.
size_t full_tc_smem_bytes(int B, bool fp8);

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel and
// device (again only to raise it): the attribute call costs host time on
// every launch otherwise.
cudaError_t set_smem_once(const void *kern, int bytes);
// cudaFuncSetAttribute(NonPortableClusterSizeAllowed) once per kernel and
// device, for clusters of more than 8 CTAs.
cudaError_t allow_wide_clusters_once(const void *kern);

// Launch with programmatic stream serialization (unless HS2_PDL=0) and an
// optional 1-D cluster.
bool pdl_enabled();
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster_x,
                      Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Cooperative launch (every CTA resident at once), with programmatic stream
// serialization as well where the runtime accepts the pair (else without it).
template <typename... KArgs, typename... Args>
cudaError_t launch_coop(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess && cfg.numAttrs == 2) {
    (void)cudaGetLastError();  // the refused pair is not the caller's error
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, args...);
  }
  return e;
}

// ---- launchers (return cudaError_t of the launch) -------------------------
cudaError_t launch_full_mma(const FullParams &p, const CUtensorMap &tmk, const CUtensorMap &tmv, bool fp8,
                            const FullMmaConfig &cfg, int grid, cudaStream_t s);
// Attention and the selection's score pass in one cooperative persistent
// launch (cudaErrorInvalidConfiguration when no fused kernel is built for cfg).
cudaError_t launch_full_fused(const FullParams &p, const ScoreParams &sp, const CUtensorMap &tmk,
                              const CUtensorMap &tmv, bool fp8, const FullMmaConfig &cfg, int grid, cudaStream_t s);
cudaError_t launch_full_f32(const FullParams &p, int grid, cudaStream_t s);
int full_f32_tile();
int full_f32_ctas_per_sm();

cudaError_t launch_select(const ScoreParams &p, cudaStream_t s);
// The filter and final kernels alone (after the fused call's score pass).
cudaError_t launch_select_after_score(const ScoreParams &p, cudaStream_t s);
// Block-level selection (first-generation comparator) in place of launch_select.
cudaError_t launch_block_select(const ScoreParams &p, int block, cudaStream_t s);

cudaError_t launch_sparse_impl(const SparseParams &p, int kv_dtype, int64_t num_slots, cudaStream_t s);

cudaError_t launch_copy(void *dst, const void *src, size_t bytes, int grid, cudaStream_t s);

cudaError_t launch_wait_selftest(uint32_t *err, cudaStream_t s);
cudaError_t launch_grid_barrier_selftest(uint32_t *err, cudaStream_t s);

// KV Bridging append of one decode step.
struct BridgeParams {
  const __nv_bfloat16 *h;            // [B, d_model]
  const __nv_bfloat16 *wk, *wv;      // [d_model, N] row-major, N = Hkv * D
  const int32_t *seq_lens;           // [B]
  const int32_t *page_table;         // [B, max_pages] or nullptr
  void *k, *v;                       // cache rows [num_slots, Hkv, D]
  float *k_scale, *v_scale;          // E4M3 only
  int32_t kv_dtype;
  int32_t B, d_model, Hkv, D, N;
  int32_t page_size, max_pages;
  int64_t t_cap, num_slots;
  int32_t nsplit;                    // row splits of d_model
  int32_t ntiles, ngroups;           // column tiles, token groups (set by launch_bridge)
  int32_t *tickets;                  // workspace [2][ntiles][ngroups], zero between calls
  float *partial;                    // workspace [2][nsplit][B][N]
};
int bridge_splits(int d_model);
int bridge_row_multiple();
size_t bridge_workspace_bytes(int B, int d_model, int N);
// Splits `workspace` into tickets and partial sums and launches the append.
cudaError_t launch_bridge(const BridgeParams &p, void *workspace, cudaStream_t s);

// Sets the thread's hs2_last_error() text and returns `code`.
int set_last_error(int code, const char *msg);

}  // namespace hs2
