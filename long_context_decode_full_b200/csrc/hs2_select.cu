// hs2_select.cu -- token-level selection of a Hybrid Block (HySparse2
// announcement: the full layer picks important positions from its attention
// scores; selection is per token; the most recent `window` tokens are always
// kept plus the top `k_global` tokens from outside that window).
//
// Score of position t for KV head j: sum over the query heads h of j's GQA
// group of softmax probability p_{h,t} = exp(c * s_{h,t} - LSE_h).
//
// Three kernels, all on the CUDA cores:
//   score  -- per (chunk, kv head, sequence): LSE of the group's heads from
//             the segment records (fp64), the final attention output of the
//             unit (chunk 0), the fp32 group score of every selectable
//             position and a 4096-bin histogram of the score's top bits; the
//             last chunk to finish (atomic ticket, no waiting) finds the bin
//             that holds the k-th largest score.
//   filter -- per chunk: positions above that bin go straight into a bitmap
//             (one warp ballot per 32 positions); positions inside it are
//             appended to a candidate list.
//   final  -- per unit: radix refinement of the candidates to the exact k-th
//             score, ties resolved to the lower position, then an ordered
//             compaction (block scans over the bitmaps) that merges the forced
//             window and writes slots in ascending position order.
// Scores are >= 0, so their IEEE bit patterns order like the values.
#include "hs2_internal.h"

namespace hs2 {

namespace {

struct UnitInfo {
  int T, nC, nb;
  int64_t U;   // first linear tile of the unit
  int nseg;
  bool select; // nC > k_global
};

__device__ __forceinline__ UnitInfo unit_info(const ScoreParams &p, int b, int kvh) {
  UnitInfo ui;
  ui.T = clamp_len(__ldg(p.seq_lens + b), (int)p.t_cap);
  ui.nC = max(0, ui.T - p.window);
  ui.select = ui.nC > p.k_global && p.k_global > 0;
  ui.nb = (ui.T + p.tile - 1) / p.tile;
  const int64_t total = (int64_t)p.Hkv * p.ws.prefix[p.B];
  ui.U = (int64_t)p.Hkv * p.ws.prefix[b] + (int64_t)kvh * ui.nb;
  ui.nseg = 0;
  if (ui.nb > 0 && total > 0) {
    const Partition part{total, p.N};
    ui.nseg = (int)(part.cfirst(ui.U + ui.nb - 1) - part.cfirst(ui.U) + 1);
    if (ui.nseg > p.R) ui.nseg = p.R;
  }
  return ui;
}

__device__ __forceinline__ int64_t slot_of(const ScoreParams &p, int b, int64_t pos) {
  if (p.page_table == nullptr) return (int64_t)b * p.page_size + pos;
  return (int64_t)__ldg(p.page_table + (int64_t)b * p.max_pages + pos / p.page_size) * p.page_size +
         pos % p.page_size;
}

// Block-wide exclusive scan of one int per thread (blockDim.x <= 1024).
__device__ __forceinline__ int block_exclusive_scan(int x, int *sh_warp, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sh_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? sh_warp[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < nw) sh_warp[lane] = wi - w;
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const int r = sh_warp[warp] + incl - x;
  __syncthreads();
  return r;
}

// Finds, over a histogram in shared memory (nbins, bin index increasing with
// score), the bin holding the need-th largest element: returns the bin and
// writes the count strictly above it.  Called by the whole block.
__device__ int find_threshold_bin(const uint32_t *hist, int nbins, int need, int *above_out, int *sh_warp,
                                  int *sh_res) {
  const int per = (nbins + blockDim.x - 1) / blockDim.x;
  if (threadIdx.x == 0) {  // defaults if the histogram holds fewer than `need`
    sh_res[0] = 0;
    sh_res[1] = 0;
  }
  // thread i owns bins counted from the top: [i*per, (i+1)*per) in descending order
  int cnt = 0;
  for (int k = 0; k < per; ++k) {
    const int bin = nbins - 1 - (threadIdx.x * per + k);
    if (bin >= 0) cnt += (int)hist[bin];
  }
  int tot;
  const int before = block_exclusive_scan(cnt, sh_warp, &tot);
  if (before < need && before + cnt >= need) {
    int acc = before;
    for (int k = 0; k < per; ++k) {
      const int bin = nbins - 1 - (threadIdx.x * per + k);
      if (bin < 0) break;
      if (acc + (int)hist[bin] >= need) {
        sh_res[0] = bin;
        sh_res[1] = acc;
        break;
      }
      acc += (int)hist[bin];
    }
  }
  __syncthreads();
  const int bin = sh_res[0];
  *above_out = sh_res[1];
  __syncthreads();
  return bin;
}

// ------------------------------------------------------------------ score
template <int G, int D>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(const ScoreParams p) {
  __shared__ uint32_t sh_hist[kHistBins];
  __shared__ double sh_lse[G];
  __shared__ float sh_M[G], sh_L[G];
  __shared__ int sh_warp[32], sh_res[2], sh_last;
  const int chunk = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const UnitInfo ui = unit_info(p, b, kvh);
  const int n_chunks = ui.select ? (ui.nC + kScoreChunk - 1) / kScoreChunk : 0;
  const bool do_out = chunk == 0;
  if (!do_out && chunk >= n_chunks) return;
  const int64_t u = (int64_t)b * p.Hkv + kvh;
  const float *rec0 = p.ws.records + (size_t)u * p.R * G * (D + 2);
  const int RS = G * (D + 2);

  // LSE of each head from the segment records: c*M + log(sum_j l_j exp(c (m_j - M)))
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int j = 0; j < ui.nseg; ++j) M = fmaxf(M, rec0[j * RS + h]);
    double L = 0.0;
    float Lf = 0.f;
    for (int j = 0; j < ui.nseg; ++j) {
      const float mj = rec0[j * RS + h];
      if (mj == -INFINITY) continue;
      const double w = exp((double)p.c * ((double)mj - (double)M));
      L += (double)rec0[j * RS + G + h] * w;
      Lf += rec0[j * RS + G + h] * expf(p.c * (mj - M));
    }
    sh_lse[h] = (double)p.c * (double)M + log(L);
    sh_M[h] = M;
    sh_L[h] = Lf;
  }
  __syncthreads();

  if (do_out) {  // out = sum_j o_j exp(c (m_j - M)) / L
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
      const int h = e / D;
      float acc = 0.f;
      for (int j = 0; j < ui.nseg; ++j) {
        const float mj = rec0[j * RS + h];
        if (mj == -INFINITY) continue;
        acc += rec0[j * RS + 2 * G + e] * expf(p.c * (mj - sh_M[h]));
      }
      const float val = ui.nseg > 0 && sh_L[h] > 0.f ? acc / sh_L[h] : 0.f;
      const int64_t oi = ((int64_t)b * p.Hkv * G + (int64_t)kvh * G) * D + e;
      if (p.out_dtype == 0) static_cast<float *>(p.out)[oi] = val;
      else static_cast<__nv_bfloat16 *>(p.out)[oi] = __float2bfloat16_rn(val);
    }
  }
  if (chunk >= n_chunks) return;

  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh_hist[i] = 0u;
  __syncthreads();
  const int t0 = chunk * kScoreChunk, t1 = min(ui.nC, t0 + kScoreChunk);
  const float *lg = p.ws.logits + (size_t)u * p.t_cap * G;
  float *sc = p.ws.scores + (size_t)u * p.t_cap;
  for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
    float raw[G];
    if constexpr (G % 4 == 0) {
#pragma unroll
      for (int h4 = 0; h4 < G / 4; ++h4) {
        const float4 v4 = __ldcs(reinterpret_cast<const float4 *>(lg + (size_t)t * G) + h4);
        raw[4 * h4] = v4.x;
        raw[4 * h4 + 1] = v4.y;
        raw[4 * h4 + 2] = v4.z;
        raw[4 * h4 + 3] = v4.w;
      }
    } else {
#pragma unroll
      for (int h = 0; h < G; ++h) raw[h] = __ldcs(lg + (size_t)t * G + h);
    }
    // p_h = exp(c*raw - LSE_h): the argument in fp64, split hi + lo, so the
    // only rounding left is expf's own
    double acc = 0.0;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const double x = (double)p.c * (double)raw[h] - sh_lse[h];
      const float xh = (float)x;
      const float xl = (float)(x - (double)xh);
      const float e = expf(xh);
      acc += (double)fmaf(e, xl, e);
    }
    const float s = acc >= 0.0 ? (float)acc : 0.f;  // NaN (bad inputs) ranks lowest
    sc[t] = s;
    atomicAdd(&sh_hist[__float_as_uint(s) >> kHistShift], 1u);
  }
  __syncthreads();
  uint32_t *gh = p.ws.hist + (size_t)u * kHistBins;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (sh_hist[i]) atomicAdd(gh + i, sh_hist[i]);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) sh_last = atomicAdd(p.ws.ticket + u, 1u) == (uint32_t)(n_chunks - 1);
  __syncthreads();
  if (!sh_last) return;
  __threadfence();
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh_hist[i] = __ldcg(gh + i);
  __syncthreads();
  int above;
  const int bin = find_threshold_bin(sh_hist, kHistBins, p.k_global, &above, sh_warp, sh_res);
  if (threadIdx.x == 0) p.ws.thr[u] = make_int2(bin, above);
}

// ------------------------------------------------------------------ filter
__global__ void __launch_bounds__(kScoreThreads) filter_kernel(const ScoreParams p) {
  const int chunk = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int T = clamp_len(__ldg(p.seq_lens + b), (int)p.t_cap);
  const int nC = max(0, T - p.window);
  if (nC <= p.k_global || p.k_global == 0 || chunk * kScoreChunk >= nC) return;
  const int64_t u = (int64_t)b * p.Hkv + kvh;
  const int2 thr = p.ws.thr[u];
  const uint32_t bin1 = (uint32_t)thr.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t words = (p.t_cap + 31) / 32;
  const float *sc = p.ws.scores + (size_t)u * p.t_cap;
  uint32_t *sel = p.ws.sel + (size_t)u * words;
  uint32_t *tie = p.ws.tie + (size_t)u * words;
  uint2 *cand = p.ws.cand + (size_t)u * p.t_cap;
  const int t0 = chunk * kScoreChunk, t1 = min(nC, t0 + kScoreChunk);
  for (int base = t0 + 32 * warp; base < t1; base += 32 * (kScoreThreads / 32)) {
    const int t = base + lane;
    const bool valid = t < t1;
    const uint32_t bits = valid ? __float_as_uint(__ldcs(sc + t)) : 0u;
    const uint32_t bin = bits >> kHistShift;
    const uint32_t above = __ballot_sync(0xffffffffu, valid && bin > bin1);
    const uint32_t eq = __ballot_sync(0xffffffffu, valid && bin == bin1);
    if (lane == 0) {
      sel[base >> 5] = above;
      tie[base >> 5] = 0u;
    }
    if (eq) {
      uint32_t pos = 0;
      if (lane == 0) pos = atomicAdd(p.ws.cand_count + u, (uint32_t)__popc(eq));
      pos = __shfl_sync(0xffffffffu, pos, 0);
      if (valid && bin == bin1) cand[pos + __popc(eq & ((1u << lane) - 1u))] = make_uint2(bits, (uint32_t)t);
    }
  }
}

// ------------------------------------------------------------------ final
__global__ void __launch_bounds__(kFinalThreads) final_kernel(const ScoreParams p) {
  __shared__ uint32_t sh_hist[2048];
  __shared__ int sh_warp[32], sh_res[2], sh_tot;
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int T = clamp_len(__ldg(p.seq_lens + b), (int)p.t_cap);
  const int nC = max(0, T - p.window);
  const int L = p.window + p.k_global;
  const int64_t u = (int64_t)b * p.Hkv + kvh;
  int32_t *idx = p.idx_out + (size_t)u * L;
  const int64_t words = (p.t_cap + 31) / 32;
  uint32_t *sel = p.ws.sel + (size_t)u * words;
  uint32_t *tie = p.ws.tie + (size_t)u * words;
  const bool all = nC <= p.k_global;
  const bool none = !all && p.k_global == 0;  // window only
  int need_eq = 0;

  if (!all && !none) {
    const uint2 *cand = p.ws.cand + (size_t)u * p.t_cap;
    const uint32_t cc = p.ws.cand_count[u];
    const int n1 = cc < (uint32_t)nC ? (int)cc : nC;
    const int2 thr = p.ws.thr[u];
    int need = p.k_global - thr.y;  // >= 1
    uint32_t prefix = (uint32_t)thr.x << kHistShift, mask = 0xFFFFFFFFu << kHistShift;
    // two refinement rounds: bits 18..8 (2048 bins), then bits 7..0 (256 bins)
    const int shifts[2] = {8, 0}, widths[2] = {11, 8};
    for (int round = 0; round < 2; ++round) {
      const int sh = shifts[round], nb = 1 << widths[round];
      for (int i = threadIdx.x; i < nb; i += blockDim.x) sh_hist[i] = 0u;
      __syncthreads();
      for (int i = threadIdx.x; i < n1; i += blockDim.x) {
        const uint32_t bits = __ldcg(&cand[i].x);
        if ((bits & mask) == prefix) atomicAdd(&sh_hist[(bits >> sh) & (nb - 1)], 1u);
      }
      __syncthreads();
      int above;
      const int bin = find_threshold_bin(sh_hist, nb, need, &above, sh_warp, sh_res);
      need -= above;
      prefix |= (uint32_t)bin << sh;
      mask |= (uint32_t)(nb - 1) << sh;
    }
    need_eq = need;  // how many positions scoring exactly `prefix` are taken
    const uint32_t kth = prefix;
    for (int i = threadIdx.x; i < n1; i += blockDim.x) {
      const uint2 cv = __ldcg(&cand[i]);
      if (cv.x > kth) atomicOr(sel + (cv.y >> 5), 1u << (cv.y & 31));
      else if (cv.x == kth) atomicOr(tie + (cv.y >> 5), 1u << (cv.y & 31));
    }
    __syncthreads();
  }

  // ordered compaction over the words of [0, T)
  const int nw = (T + 31) / 32;
  const int per = (nw + blockDim.x - 1) / blockDim.x;
  const int w0 = min(nw, threadIdx.x * per), w1 = min(nw, w0 + per);
  auto cmask = [&](int w) -> uint32_t {  // bits of selectable positions (< nC)
    const int lo = w * 32;
    if (lo + 32 <= nC) return 0xFFFFFFFFu;
    if (lo >= nC) return 0u;
    return (1u << (nC - lo)) - 1u;
  };
  auto tmask = [&](int w) -> uint32_t {  // bits of positions < T
    const int lo = w * 32;
    if (lo + 32 <= T) return 0xFFFFFFFFu;
    return (1u << (T - lo)) - 1u;
  };
  int tie_before = 0;
  if (!all && !none) {
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(__ldcg(tie + w) & cmask(w));
    tie_before = block_exclusive_scan(cnt, sh_warp, &sh_tot);
  }
  auto word_sel = [&](int w, int &ties_seen) -> uint32_t {
    const uint32_t cm = cmask(w), tm = tmask(w);
    if (all) return tm;
    if (none) return tm & ~cm;
    uint32_t x = (__ldcg(sel + w) & cm) | (tm & ~cm);
    uint32_t tw = __ldcg(tie + w) & cm;
    while (tw) {
      const uint32_t lowbit = tw & (0u - tw);
      if (ties_seen < need_eq) x |= lowbit;
      ++ties_seen;
      tw ^= lowbit;
    }
    return x;
  };
  int cnt = 0;
  {
    int ts = tie_before;
    for (int w = w0; w < w1; ++w) cnt += __popc(word_sel(w, ts));
  }
  const int out_before = block_exclusive_scan(cnt, sh_warp, &sh_tot);
  const int n_total = sh_tot;
  {
    int ts = tie_before, o = out_before;
    for (int w = w0; w < w1; ++w) {
      uint32_t x = word_sel(w, ts);
      while (x) {
        const int bit = __ffs(x) - 1;
        x &= x - 1;
        if (o < L) idx[o] = (int32_t)slot_of(p, b, (int64_t)w * 32 + bit);
        ++o;
      }
    }
  }
  for (int i = n_total + threadIdx.x; i < L; i += blockDim.x) idx[i] = -1;
}

template <int G>
cudaError_t launch_score_g(const ScoreParams &p, dim3 grid, cudaStream_t s) {
  if (p.D == 64) score_kernel<G, 64><<<grid, kScoreThreads, 0, s>>>(p);
  else score_kernel<G, 128><<<grid, kScoreThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const ScoreParams &p, cudaStream_t s) {
  const int chunks = (int)((p.t_cap + kScoreChunk - 1) / kScoreChunk);
  const dim3 grid(max(chunks, 1), p.Hkv, p.B);
  cudaError_t e;
  switch (p.G) {
    case 1: e = launch_score_g<1>(p, grid, s); break;
    case 2: e = launch_score_g<2>(p, grid, s); break;
    case 4: e = launch_score_g<4>(p, grid, s); break;
    case 8: e = launch_score_g<8>(p, grid, s); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  filter_kernel<<<grid, kScoreThreads, 0, s>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  final_kernel<<<dim3(p.Hkv, p.B), kFinalThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace hs2
