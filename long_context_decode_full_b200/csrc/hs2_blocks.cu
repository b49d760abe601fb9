// hs2_blocks.cu -- block-level selection, the first-generation HySparse
// comparator (HySparse2 announcement, the paragraphs contrasting token-level
// selection with HySparse's block-level one: v1 chose whole blocks, so an
// important token brought the block around it with it; HySparse2 chooses
// tokens, and the two were compared at the same token budget).
//
// Readings where the pages are silent: the selectable positions [0, T - W)
// are cut into blocks [j block, (j + 1) block), the last one cut short at
// T - W; a block's score is the sum of its positions' group scores (the same
// group score as the token-level path); k_global / block blocks are taken by
// (block score descending, block index ascending), all of them when there are
// no more; the forced window [T - W, T) is always taken.  The index list holds
// the slots of the taken positions in position order, -1 padded.
//
// Two kernels after the attention pass:
//   block_score  -- grid (chunk, kv head, sequence) + combine CTAs: the exact
//                   group score of every selectable position (exponent in
//                   float-float, ~2^-22 relative), and the attention output.
//   block_select -- one CTA per unit: block sums in fp64, a 4096-bin
//                   histogram of their fp32 values for the threshold block,
//                   a radix select on the fp64 bits among the blocks of the
//                   threshold bin (ties to the lower block), then the kept
//                   blocks' positions in order, followed by the window.
#include "hs2_internal.h"
#include "hs2_select_common.cuh"

namespace hs2 {

namespace {

template <int G, int D>
__global__ void __launch_bounds__(kScoreThreads) block_score_kernel(const ScoreParams p) {
  __shared__ uint32_t sh_hist[kHistBins];  // the combine CTAs' weights
  __shared__ double sh_red[kScoreThreads];
  __shared__ double sh_lse[G];
  __shared__ float sh_M[G], sh_L[G];
  __shared__ uint8_t sh_ok[kMaxRecords];
  constexpr int RS = G * (D + 2);
  griddep_wait();
  griddep_launch_dependents();
  const int chunk = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int comb = chunk - ((int)gridDim.x - p.ncomb);
  const bool combine = comb >= 0;
  UnitInfo ui = unit_info(p, b, kvh);
  const int t0 = chunk * p.score_chunk, t1 = min(ui.nC, t0 + p.score_chunk);
  if (!combine && t0 >= ui.nC) return;
  const int64_t u = (int64_t)b * p.Hkv + kvh;
  mark_records(ui, sh_ok);
  unit_lse<G, D>(p.ws.records + (size_t)u * p.R * RS, ui, p.c, sh_lse, sh_M, sh_L, sh_red);
  if (combine) {
    combine_unit<G, D>(p, ui, u, comb, sh_M, sh_L, sh_hist);
    return;
  }
  const float *lg = p.ws.logits + (size_t)u * p.ustride * G;
  float *sc = p.ws.scores + (size_t)u * p.ustride;
  for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) sc[t] = exact_score(lg + (size_t)t * G, G, p.c, sh_lse);
}

__device__ __forceinline__ uint32_t f32_bin(double s) {
  const float f = (float)s;
  return (f >= 0.f ? __float_as_uint(f) : 0u) >> kHistShift;  // (NaN ranks lowest)
}
__device__ __forceinline__ uint64_t f64_bits(double s) {
  return s >= 0.0 ? (uint64_t)__double_as_longlong(s) : 0ull;  // non-negative: bits order like values
}

// One CTA (kFinalThreads) per unit.  Dynamic shared memory: the kept block
// indices, kMaxSelect ints.
__global__ void __launch_bounds__(kFinalThreads) block_select_kernel(const ScoreParams p, int block) {
  extern __shared__ int kept[];
  __shared__ uint32_t sh_hist[kHistBins];
  __shared__ int sh_warp[33], sh_res[2];
  griddep_wait();
  griddep_launch_dependents();
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int T = clamp_len(__ldg(p.seq_lens + b), (int)p.t_cap);
  const int nC = max(0, T - p.window);
  const int L = p.window + p.k_global;
  const int64_t u = (int64_t)b * p.Hkv + kvh;
  int32_t *idx = p.idx_out + (size_t)u * L;
  const int nblk = (nC + block - 1) / block, keep = p.k_global / block;
  const float *sc = p.ws.scores + (size_t)u * p.ustride;
  double *bs = reinterpret_cast<double *>(p.ws.cand) + (size_t)u * p.ustride;  // block sums (<= 8 B per position)
  int n_sel;  // selectable positions taken (before the window)
  if (keep == 0) {
    n_sel = 0;
  } else if (nblk <= keep) {
    n_sel = nC;
    for (int t = threadIdx.x; t < nC; t += blockDim.x) idx[t] = (int32_t)slot_of(p, b, t);
  } else {
    // block sums in fp64 (positions in order) and the histogram of their fp32 values
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh_hist[i] = 0u;
    __syncthreads();
    for (int j = threadIdx.x; j < nblk; j += blockDim.x) {
      const int ta = j * block, tb = min(ta + block, nC);
      double s = 0.0;
      for (int t = ta; t < tb; ++t) s += (double)sc[t];
      bs[j] = s;
      atomicAdd(&sh_hist[f32_bin(s)], 1u);
    }
    __syncthreads();
    int above;
    const uint32_t bin = (uint32_t)find_threshold_bin(sh_hist, kHistBins, keep, &above, sh_warp, sh_res);
    // the need-th largest fp64 block sum inside the threshold bin: radix select
    // on its bit pattern, 11 bits a round from the top
    int rem = keep - above;
    uint64_t prefix = 0ull, mask = 0ull;
    const int shifts[6] = {53, 42, 31, 20, 9, 0}, widths[6] = {11, 11, 11, 11, 11, 9};
    for (int round = 0; round < 6; ++round) {
      const int sh = shifts[round], nb = 1 << widths[round];
      for (int i = threadIdx.x; i < nb; i += blockDim.x) sh_hist[i] = 0u;
      __syncthreads();
      for (int j = threadIdx.x; j < nblk; j += blockDim.x) {
        const double s = bs[j];
        const uint64_t x = f64_bits(s);
        if (f32_bin(s) == bin && (x & mask) == prefix) atomicAdd(&sh_hist[(x >> sh) & (uint64_t)(nb - 1)], 1u);
      }
      __syncthreads();
      int ab;
      const int rb = find_threshold_bin(sh_hist, nb, rem, &ab, sh_warp, sh_res);
      rem -= ab;
      prefix |= (uint64_t)rb << sh;
      mask |= (uint64_t)(nb - 1) << sh;
    }
    __syncthreads();
    const uint64_t kth = prefix;  // keep `rem` of its ties, the lowest blocks first
    // kept blocks in index order: above the bin, or in the bin and above the
    // k-th sum, or one of its first `rem` ties
    int nkept = 0, ties = 0;
    for (int base = 0; base < nblk; base += blockDim.x) {
      const int j = base + threadIdx.x;
      int take = 0, tie = 0;
      if (j < nblk) {
        const double s = bs[j];
        const uint32_t fb = f32_bin(s);
        const uint64_t x = f64_bits(s);
        tie = fb == bin && x == kth;
        take = fb > bin || (fb == bin && x > kth);
      }
      int tie_tot;
      const int tie_rank = ties + block_exclusive_scan(tie, sh_warp, &tie_tot);
      ties += tie_tot;
      take |= tie && tie_rank < rem;
      int tot;
      const int pos = nkept + block_exclusive_scan(take, sh_warp, &tot);
      if (take && pos < kMaxSelect) kept[pos] = j;
      nkept += tot;
    }
    __syncthreads();
    nkept = min(nkept, keep);
    // positions of the kept blocks, in order; only the last block can be short
    n_sel = 0;
    if (nkept > 0) n_sel = (nkept - 1) * block + (min((kept[nkept - 1] + 1) * block, nC) - kept[nkept - 1] * block);
    for (int e = threadIdx.x; e < n_sel; e += blockDim.x) {
      const int t = kept[e / block] * block + e % block;
      if (e < L) idx[e] = (int32_t)slot_of(p, b, t);
    }
  }
  // the forced window follows every selectable position taken
  for (int t = nC + threadIdx.x; t < T; t += blockDim.x) {
    const int o = n_sel + (t - nC);
    if (o < L) idx[o] = (int32_t)slot_of(p, b, t);
  }
  for (int i = n_sel + (T - nC) + threadIdx.x; i < L; i += blockDim.x) idx[i] = -1;
}

template <int G>
cudaError_t launch_block_score_g(const ScoreParams &p, dim3 grid, cudaStream_t s) {
  if (p.D == 64) return launch_ex(block_score_kernel<G, 64>, grid, dim3(kScoreThreads), 0, s, 0, p);
  return launch_ex(block_score_kernel<G, 128>, grid, dim3(kScoreThreads), 0, s, 0, p);
}

}  // namespace

cudaError_t launch_block_select(const ScoreParams &p, int block, cudaStream_t s) {
  const int chunks = (int)((p.t_cap + p.score_chunk - 1) / p.score_chunk);
  const dim3 grid(chunks + p.ncomb, p.Hkv, p.B);
  cudaError_t e;
  switch (p.G) {
    case 1: e = launch_block_score_g<1>(p, grid, s); break;
    case 2: e = launch_block_score_g<2>(p, grid, s); break;
    case 4: e = launch_block_score_g<4>(p, grid, s); break;
    case 8: e = launch_block_score_g<8>(p, grid, s); break;
    case 16: e = launch_block_score_g<16>(p, grid, s); break;
    case 32: e = launch_block_score_g<32>(p, grid, s); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)kMaxSelect * sizeof(int);
  return launch_ex(block_select_kernel, dim3(p.Hkv, p.B), dim3(kFinalThreads), smem, s, 0, p, block);
}

}  // namespace hs2
