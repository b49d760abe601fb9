// hs2_sparse.cu -- a sparse-attention layer of a Hybrid Block (HySparse2
// announcement, "KV Reuse" section: the sparse layers reuse the full layer's
// KV cache and its selection indices; the forced window and the global
// tokens are read from that one cache in a single sparse computation, with
// no separate sliding-window branch).
//
// Per (sequence, kv head) a thread-block cluster of `splits` CTAs shares the
// index list: every warp gathers 16 listed rows of K and V (whole rows,
// 16-byte cp.async into the swizzled tile layout), runs the tensor-core
// attention step for the G query heads of the group, the CTA merges its
// warps, and the CTAs merge through distributed shared memory, each writing
// its share of the output elements.  No workspace, no atomics, one launch.
// fp32 caches take the same cluster shape on the CUDA cores (FFMA): 64-row
// tiles gathered with 4-byte cp.async, one warp per query head.
#include <cooperative_groups.h>

#include "hs2_internal.h"
#include "hs2_warp_attn.cuh"

namespace cg = cooperative_groups;

namespace hs2 {

namespace {

// NW warps per CTA, each taking groups of RG = 16 NSL listed rows (NSL
// 16-row slices per tensor-core step).
template <int D, bool FP8, int NW, int NSL>
struct SCfg {
  static constexpr int RG = 16 * NSL;                               // rows per group
  static constexpr int ES = FP8 ? 1 : 2;
  static constexpr int ROWB = D * ES;
  static constexpr int PANEL = RG * 128;
  static constexpr int KVB = RG * ROWB;                             // RG rows of K (or V)
  static constexpr int BUF_BYTES = 2 * KVB + (FP8 ? 2 * RG * 4 : 0);  // one group
  static constexpr int WSTRIDE = 16 + 8 * D;                        // warp scratch floats
  // one CTA's partial record m[G], l[G], o[G][D], padded to whole float4s
  __host__ __device__ static int rec_floats(int G) { return (G * (D + 2) + 3) & ~3; }
  __host__ __device__ static size_t staging(int nbuf) { return (size_t)NW * nbuf * BUF_BYTES; }
  // the warps' merge scratch reuses the staging buffers (idle by then) when
  // it fits, else gets a region of their own
  __host__ __device__ static size_t scratch_bytes(int, int) { return (size_t)NW * WSTRIDE * 4; }
  __host__ __device__ static bool scratch_in_staging(int G, int S, int nbuf) {
    return scratch_bytes(G, S) <= staging(nbuf);
  }
  static size_t bytes(int G, int S, int rows, int nbuf) {  // G: heads of one cluster (<= 8)
    return 128 + staging(nbuf) + (scratch_in_staging(G, S, nbuf) ? 0 : scratch_bytes(G, S)) +
           (size_t)rec_floats(G) * 4 + (size_t)(3 * S + 1) * 8 * 4 + (size_t)rows * 4;
  }
};

__device__ __forceinline__ void cp_async_wait_n(int n) {  // n = groups allowed to stay pending (<= 3)
  if (n <= 0) asm volatile("cp.async.wait_group 0;" ::: "memory");
  else if (n == 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
  else if (n == 2) asm volatile("cp.async.wait_group 2;" ::: "memory");
  else asm volatile("cp.async.wait_group 3;" ::: "memory");
}

// Grid (splits, Hkv, B), cluster (splits, 1, 1), 8 warps.  CTA `rank` of a
// unit's cluster owns rows [rank * rows_per_cta, ...) of the index list; its
// warps take 16-row groups round-robin.  Each warp issues the gathers of up
// to `nbuf` groups at once, so their latencies overlap, and computes each
// group on the tensor cores as it lands.
template <int D, bool FP8, int NW, int NSL>
__global__ void __launch_bounds__(32 * NW, 1) sparse_mma_kernel(const SparseParams p, int64_t num_slots) {
  using C = SCfg<D, FP8, NW, NSL>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  cg::cluster_group cluster = cg::this_cluster();
  const int S = (int)cluster.num_blocks();
  const int Gc = p.G < 8 ? p.G : 8;  // heads of one cluster (the shared-memory layout)
  const int RSP = C::rec_floats(Gc);
  const int nbuf = p.nbuf;
  const bool in_staging = C::scratch_in_staging(Gc, S, nbuf);
  uint8_t *after = smem + C::staging(nbuf) + (in_staging ? 0 : C::scratch_bytes(p.G, S));
  float *scratch = reinterpret_cast<float *>(in_staging ? smem : smem + C::staging(nbuf));
  float *partial = reinterpret_cast<float *>(after);             // m[G], l[G], o[G][D] of this CTA
  float *wts = partial + RSP;                                    // weight of (CTA, head)
  float *inv_l = wts + S * 8;                                    // 1 / normaliser per head
  float *ms_ = inv_l + 8, *ls_ = ms_ + S * 8;                    // (m, l) of (CTA, head)
  int *slots = reinterpret_cast<int *>(ls_ + S * 8);             // this CTA's index entries
  const int rank = (int)cluster.block_rank();
  // blockIdx.y = (kv head, group of 8 query heads): groups above 8 heads
  // (MQA-style) take one cluster per 8 heads, each gathering the rows itself
  const int nhg = (p.G + 7) >> 3;
  const int kvh = blockIdx.y / nhg, hg = blockIdx.y % nhg, b = blockIdx.z;
  const int G = min(8, p.G - 8 * hg);  // heads of this cluster
  const int64_t u = (int64_t)b * p.Hkv + kvh;
  const int64_t head0 = (int64_t)b * p.Hkv * p.G + (int64_t)kvh * p.G + 8 * hg;  // first query head
  const int row_lo = rank * p.rows_per_cta, nrows = max(0, min(p.L, row_lo + p.rows_per_cta) - row_lo);
  griddep_wait();  // the index list and the query come from earlier kernels
  griddep_launch_dependents();

  // the CTA's slice of the index list, validated (entries outside the cache are skipped)
  for (int r = threadIdx.x; r < nrows; r += blockDim.x) {
    const int sl = __ldg(p.idx + u * p.L + row_lo + r);
    slots[r] = (sl >= 0 && sl < num_slots) ? sl : -1;
  }
  WarpAttn<D, FP8, NSL> st;
  st.reset();
  st.load_q(static_cast<const __nv_bfloat16 *>(p.q) + head0 * D, G);
  __syncthreads();

  constexpr int CPR = C::ROWB / 16;  // 16-byte chunks per row
  const uint8_t *kg = static_cast<const uint8_t *>(p.k), *vg = static_cast<const uint8_t *>(p.v);
  uint8_t *wbase = smem + (size_t)warp * nbuf * C::BUF_BYTES;
  // issue the loads of RG-row group `grp` into buffer `buf`; returns its row mask
  auto gather = [&](int grp, int buf) -> uint32_t {
    uint8_t *wb = wbase + buf * C::BUF_BYTES;
    const uint32_t kp = smem_u32(wb), vp = kp + C::KVB;
    const int r = C::RG * grp + (lane & (C::RG - 1));
    const int slot = r < nrows ? slots[r] : -1;
    const uint32_t vm = __ballot_sync(0xffffffffu, slot >= 0) & (C::RG == 32 ? 0xFFFFFFFFu : 0xFFFFu);
    if constexpr (FP8) {
      float *ks = reinterpret_cast<float *>(wb + 2 * C::KVB);
      if (lane < C::RG) {
        if (slot >= 0) {
          cp_async_4(smem_u32(ks + lane), p.k_scale + (int64_t)slot * p.Hkv + kvh);
          cp_async_4(smem_u32(ks + C::RG + lane), p.v_scale + (int64_t)slot * p.Hkv + kvh);
        } else {
          ks[lane] = 0.f;
          ks[C::RG + lane] = 0.f;
        }
      }
    }
#pragma unroll 4
    for (int e = lane; e < C::RG * CPR; e += 32) {
      const int row = e / CPR, ch = e % CPR;
      const int sr = __shfl_sync(0xffffffffu, slot, row);
      const uint32_t off = (ch >> 3) * C::PANEL;
      const uint32_t dk = swz(kp + off, row, ch & 7), dv = swz(vp + off, row, ch & 7);
      if (sr >= 0) {
        const int64_t src = ((int64_t)sr * p.Hkv + kvh) * C::ROWB + ch * 16;
        cp_async_16(dk, kg + src);
        cp_async_16(dv, vg + src);
      } else {
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dk), "r"(0u) : "memory");
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dv), "r"(0u) : "memory");
      }
    }
    cp_async_commit();
    return vm;
  };

  const int ngroups = (nrows + C::RG - 1) / C::RG;
  const int mine = ngroups > warp ? (ngroups - warp + NW - 1) / NW : 0;  // groups of this warp
  uint32_t vm[4] = {0u, 0u, 0u, 0u};
  int issued = 0;
  for (; issued < mine && issued < nbuf; ++issued) vm[issued & 3] = gather(warp + issued * NW, issued % nbuf);
  for (int k = 0; k < mine; ++k) {
    cp_async_wait_n(issued - k - 1);
    __syncwarp();
    uint8_t *wb = wbase + (k % nbuf) * C::BUF_BYTES;
    const uint32_t kp = smem_u32(wb);
    const float *ks = reinterpret_cast<const float *>(wb + 2 * C::KVB);
    const uint32_t m = vm[k & 3];
    if (m) st.step(kp, kp + C::KVB, C::PANEL, 0, m, p.c, nullptr, G, ks, ks + C::RG);
    __syncwarp();  // the buffer is refilled by the next gather
    if (issued < mine) {
      vm[issued & 3] = gather(warp + issued * NW, issued % nbuf);
      ++issued;
    }
  }
  cp_async_wait_all();
  __syncthreads();  // every warp is done with the staging buffers

  // ---- merge the warps of this CTA, then the CTAs of the cluster
  float *scr = scratch + warp * C::WSTRIDE;
  st.store(scr, scr + 8, scr + 16);
  __syncthreads();
  merge_warp_states<D>(scratch, C::WSTRIDE, NW, G, p.c, partial, threadIdx.x, blockDim.x);
  cluster.sync();  // every CTA's partial is complete
  // every CTA writes its share of the G x D outputs: the (m, l) pairs of all
  // partials (one per thread), the heads' weights, then its elements with the
  // partials' o read straight from the other CTAs' shared memory
  if (threadIdx.x < S * 8) {
    const int r = threadIdx.x >> 3, h = threadIdx.x & 7;
    const float *pr = cluster.map_shared_rank(partial, r);
    ms_[threadIdx.x] = h < G ? pr[h] : -INFINITY;
    ls_[threadIdx.x] = h < G ? pr[G + h] : 0.f;
  }
  __syncthreads();
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int r = 0; r < S; ++r) M = fmaxf(M, ms_[r * 8 + h]);
    float L = 0.f;
    for (int r = 0; r < S; ++r) {
      const float mr = ms_[r * 8 + h];
      const float w = mr == -INFINITY ? 0.f : expf(p.c * (mr - M));
      wts[r * 8 + h] = w;
      L += w * ls_[r * 8 + h];
    }
    inv_l[h] = L > 0.f ? 1.f / L : 0.f;
  }
  __syncthreads();
  {
    const int per = (G * D + S - 1) / S, e0 = rank * per, e1 = min(G * D, e0 + per);
    const int64_t ob = head0 * D;
    for (int e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
      const int h = e / D;
      float acc = 0.f;
      for (int r = 0; r < S; ++r) acc += wts[r * 8 + h] * cluster.map_shared_rank(partial, r)[2 * G + e];
      static_cast<__nv_bfloat16 *>(p.out)[ob + e] = __float2bfloat16_rn(acc * inv_l[h]);
    }
  }
  cluster.sync();  // keep every CTA's shared memory alive until all have read it
}

// ------------------------------------------------------------ fp32 caches
// A cluster of S CTAs (4 warps each) per (sequence, kv head): CTA r takes the
// 64-row tiles [r * ntiles / S, (r + 1) * ntiles / S) of the index list.  A
// tile's listed rows are gathered into shared memory (coalesced row loads),
// then warp w serves the heads w and w + 4 of the group with an online softmax
// on the CUDA cores (FFMA keeps fp32 logits exact to fp32 rounding).  The CTAs'
// (m, l, o) meet through distributed shared memory: each CTA writes 1/S of the
// group's G x D outputs.
constexpr int kSpF32Tile = 64;
constexpr int kSpF32Warps = 4;
constexpr int kSpF32MaxSplits = 16;

template <int D>
constexpr int sp_f32_floats() {  // shared floats before the tile's slot list
  return 2 * kSpF32Tile * (D + 1) + 8 * D + (16 + 8 * D) + 8 * kSpF32MaxSplits + 8;
}

template <int D>
__global__ void __launch_bounds__(32 * kSpF32Warps) sparse_f32_kernel(const SparseParams p, int64_t num_slots) {
  extern __shared__ float fsm[];
  float *Ks = fsm;                          // [64][D + 1]
  float *Vs = Ks + kSpF32Tile * (D + 1);    // [64][D + 1]
  float *Qs = Vs + kSpF32Tile * (D + 1);    // [G <= 8][D]
  float *part = Qs + 8 * D;                 // this CTA's m[8], l[8], o[8][D]
  float *wts = part + 16 + 8 * D;           // [rank][8] weights of the partials
  float *inv_l = wts + 8 * kSpF32MaxSplits; // [8]
  int *slots = reinterpret_cast<int *>(inv_l + 8);  // [64]
  cg::cluster_group cluster = cg::this_cluster();
  const int S = (int)cluster.num_blocks(), rank = (int)cluster.block_rank();
  const int kvh = blockIdx.y, b = blockIdx.z, G = p.G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nthr = blockDim.x;
  griddep_wait();
  griddep_launch_dependents();
  const float *q = static_cast<const float *>(p.q) + ((int64_t)b * p.Hkv * G + (int64_t)kvh * G) * D;
  for (int e = threadIdx.x; e < G * D; e += nthr) cp_async_4(smem_u32(Qs + e), q + e);  // waited on with the first tile
  const float *K = static_cast<const float *>(p.k), *V = static_cast<const float *>(p.v);
  const int32_t *idx = p.idx + ((int64_t)b * p.Hkv + kvh) * p.L;
  float m[2], l[2], o[2][D / 32];
#pragma unroll
  for (int hs = 0; hs < 2; ++hs) {
    m[hs] = -INFINITY;
    l[hs] = 0.f;
#pragma unroll
    for (int j = 0; j < D / 32; ++j) o[hs][j] = 0.f;
  }
  const int ntiles = (p.L + kSpF32Tile - 1) / kSpF32Tile;
  const int tile0 = rank * ntiles / S, tile1 = (rank + 1) * ntiles / S;
  for (int tile = tile0; tile < tile1; ++tile) {
    const int base = tile * kSpF32Tile;
    for (int r = threadIdx.x; r < kSpF32Tile; r += nthr) {
      const int sl = base + r < p.L ? __ldg(idx + base + r) : -1;
      slots[r] = (sl >= 0 && sl < num_slots) ? sl : -1;
    }
    __syncthreads();
    // every element of the tile's K and V rows in flight at once (4-byte
    // cp.async into the padded rows)
#pragma unroll 8
    for (int e = threadIdx.x; e < kSpF32Tile * D; e += 32 * kSpF32Warps) {
      const int rr = e / D, col = e % D;
      const int sl = slots[rr];
      float *kd = Ks + rr * (D + 1) + col, *vd = Vs + rr * (D + 1) + col;
      if (sl >= 0) {
        cp_async_4(smem_u32(kd), K + ((int64_t)sl * p.Hkv + kvh) * D + col);
        cp_async_4(smem_u32(vd), V + ((int64_t)sl * p.Hkv + kvh) * D + col);
      } else {
        *kd = 0.f;
        *vd = 0.f;
      }
    }
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
      const int h = warp + kSpF32Warps * hs;
      if (h >= G) break;
      float s[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int rr = lane + 32 * j;
        float acc = 0.f;
#pragma unroll 4
        for (int e = 0; e < D; ++e) acc = fmaf(Qs[h * D + e], Ks[rr * (D + 1) + e], acc);
        s[j] = slots[rr] >= 0 ? acc : -INFINITY;
      }
      const float mx = warp_max(fmaxf(s[0], s[1]));
      if (mx == -INFINITY) continue;  // no listed row in this tile
      const float m_new = fmaxf(m[hs], mx);
      const float alpha = expf(p.c * (m[hs] - m_new));
      float pr[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) pr[j] = s[j] == -INFINITY ? 0.f : expf(p.c * (s[j] - m_new));
      l[hs] = l[hs] * alpha + warp_sum(pr[0] + pr[1]);
      m[hs] = m_new;
#pragma unroll
      for (int j = 0; j < D / 32; ++j) {
        float acc = o[hs][j] * alpha;
#pragma unroll 4
        for (int rr = 0; rr < kSpF32Tile; ++rr) {
          const float pp = __shfl_sync(0xffffffffu, pr[rr >> 5], rr & 31);
          acc = fmaf(pp, Vs[rr * (D + 1) + lane + 32 * j], acc);
        }
        o[hs][j] = acc;
      }
    }
    __syncthreads();  // the tile is consumed before the next gather
  }
  cp_async_wait_all();  // (the query's copies, should this CTA have had no tile)
  // this CTA's partial state (m = -inf, l = 0 where it saw no listed row)
#pragma unroll
  for (int hs = 0; hs < 2; ++hs) {
    const int h = warp + kSpF32Warps * hs;
    if (h >= G) break;
    if (lane == 0) {
      part[h] = m[hs];
      part[8 + h] = l[hs];
    }
#pragma unroll
    for (int j = 0; j < D / 32; ++j) part[16 + h * D + lane + 32 * j] = o[hs][j];
  }
  cluster.sync();  // every CTA's partial is complete
  if (threadIdx.x < G) {  // the partials' weights per head: exp(c (m_r - M)), and 1 / sum_r w_r l_r
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int r = 0; r < S; ++r) M = fmaxf(M, cluster.map_shared_rank(part, r)[h]);
    float L = 0.f;
    for (int r = 0; r < S; ++r) {
      const float *pr = cluster.map_shared_rank(part, r);
      const float w = pr[h] == -INFINITY ? 0.f : expf(p.c * (pr[h] - M));
      wts[r * 8 + h] = w;
      L += w * pr[8 + h];
    }
    inv_l[h] = L > 0.f ? 1.f / L : 0.f;
  }
  __syncthreads();
  {  // this CTA's share of the outputs, the partials added in rank order
    const int per = (G * D + S - 1) / S, e0 = rank * per, e1 = min(G * D, e0 + per);
    float *out = static_cast<float *>(p.out) + ((int64_t)b * p.Hkv * G + (int64_t)kvh * G) * D;
    for (int e = e0 + threadIdx.x; e < e1; e += nthr) {
      const int h = e / D;
      float acc = 0.f;
      for (int r = 0; r < S; ++r) acc += wts[r * 8 + h] * cluster.map_shared_rank(part, r)[16 + e];
      out[e] = acc * inv_l[h];
    }
  }
  cluster.sync();  // keep every CTA's shared memory alive until all have read it
}

template <int D>
cudaError_t launch_f32_t(const SparseParams &p, int64_t num_slots, cudaStream_t s) {
  const size_t smem = (size_t)sp_f32_floats<D>() * 4 + kSpF32Tile * 4;
  auto kern = sparse_f32_kernel<D>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  if (p.splits > 8) {
    e = allow_wide_clusters_once(reinterpret_cast<const void *>(kern));
    if (e != cudaSuccess) return e;
  }
  return launch_ex(kern, dim3(p.splits, p.Hkv, p.B), dim3(32 * kSpF32Warps), smem, s, p.splits, p, num_slots);
}

template <int D, bool FP8, int NW, int NSL>
cudaError_t launch_mma_t(const SparseParams &p, int64_t num_slots, cudaStream_t s) {
  using C = SCfg<D, FP8, NW, NSL>;
  const size_t smem = C::bytes(p.G < 8 ? p.G : 8, p.splits, p.rows_per_cta, p.nbuf);
  auto kern = sparse_mma_kernel<D, FP8, NW, NSL>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  if (p.splits > 8) {
    e = allow_wide_clusters_once(reinterpret_cast<const void *>(kern));
    if (e != cudaSuccess) return e;
  }
  return launch_ex(kern, dim3(p.splits, p.Hkv * ((p.G + 7) / 8), p.B), dim3(32 * NW), smem, s, p.splits, p, num_slots);
}

template <int D, bool FP8>
cudaError_t launch_mma_shape(const SparseParams &p, int64_t num_slots, cudaStream_t s) {
  if (p.warps == 8 && p.nsl == 1) return launch_mma_t<D, FP8, 8, 1>(p, num_slots, s);
  if (p.warps == 4 && p.nsl == 2) return launch_mma_t<D, FP8, 4, 2>(p, num_slots, s);
  if (p.warps == 8 && p.nsl == 2) return launch_mma_t<D, FP8, 8, 2>(p, num_slots, s);
  if (p.warps == 4 && p.nsl == 1) return launch_mma_t<D, FP8, 4, 1>(p, num_slots, s);
  return cudaErrorInvalidConfiguration;
}

}  // namespace

cudaError_t launch_sparse_impl(const SparseParams &p, int kv_dtype, int64_t num_slots, cudaStream_t s) {
  if (kv_dtype == 0) {  // p.splits CTAs per (sequence, kv head), 1 .. 16
    if (p.splits < 1 || p.splits > kSpF32MaxSplits) return cudaErrorInvalidValue;
    return p.D == 64 ? launch_f32_t<64>(p, num_slots, s) : launch_f32_t<128>(p, num_slots, s);
  }
  if (kv_dtype == 1)
    return p.D == 64 ? launch_mma_shape<64, false>(p, num_slots, s) : launch_mma_shape<128, false>(p, num_slots, s);
  if (kv_dtype == 2 && p.D == 128) return launch_mma_shape<128, true>(p, num_slots, s);
  return cudaErrorInvalidValue;
}

}  // namespace hs2
