// hs2_select_common.cuh -- pieces shared by the token-level selection
// (hs2_select.cu) and the block-level comparator (hs2_blocks.cu): a unit's
// place in the attention pass's partition, its per-head log-sum-exp from the
// segment records, the combine of the records into the attention output,
// block-wide scans, the histogram threshold and the exact group score.
#pragma once

#include "hs2_internal.h"

namespace hs2 {

namespace {

constexpr double kLog2e = 1.4426950408889634074;
constexpr double kLn2 = 0.69314718055994530942;

// Far below the window, group probabilities can fall under fp32's normal
// range (2^-126: logit margins above ~87 nats), where ex2 flushes them to 0.
// When the k_global-th approximate score lies below 2^-96, the unit's scores
// are recomputed with a common factor 2^E (a common factor keeps the order):
// E is raised until the threshold bin sits near 2^-32, far from both ends of
// fp32's range.  Scores far above it may overflow to +inf; they are certainly
// selected and are counted as such.  E stops at 948, where a score still 0 in
// fp32 is below 2^-1074 and so 0 in fp64 as well.
constexpr int kTrustBin = 31 << 4;     // threshold bin of 2^-96 (biased exponent 31)
constexpr int kTargetExponent = 95;    // biased exponent of 2^-32
constexpr double kMaxShift = 948.0;

constexpr int kMaxRecords = 1024;  // >= records per unit (4 * SMs / Hkv + 2)
constexpr int kCombineElems = 256;  // output elements per combine CTA (one per thread)
// e0 is a multiple of 256, so a combine CTA covers 256 / D whole heads (at most 4 with D = 64)
static_assert(kMaxRecords * (kCombineElems / 64) <= kHistBins, "combine weights fit in the histogram");

struct UnitInfo {
  int T, nC, nb;
  int64_t U;   // first linear tile of the unit
  int64_t c0;  // CTA owning the unit's first tile: record j was written by CTA c0 + j
  int nseg;
  bool select;  // nC > k_global > 0
  Partition part;
  const uint8_t *ok;  // shared: ok[j] = record j holds a segment (its CTA owned tiles)
  __device__ __forceinline__ bool rec_ok(int j) const { return ok[j] != 0; }
};

// Marks which of the unit's record slots were written (whole block).
__device__ __forceinline__ void mark_records(UnitInfo &ui, uint8_t *sh_ok) {
  for (int j = threadIdx.x; j < ui.nseg; j += blockDim.x) sh_ok[j] = ui.part.owns_tiles(ui.c0 + j) ? 1 : 0;
  ui.ok = sh_ok;
  __syncthreads();
}

__device__ __forceinline__ UnitInfo unit_info(const ScoreParams &p, int b, int kvh) {
  UnitInfo ui;
  ui.T = clamp_len(__ldg(p.seq_lens + b), (int)p.t_cap);
  ui.nC = max(0, ui.T - p.window);
  ui.select = ui.nC > p.k_global && p.k_global > 0;
  ui.nb = (ui.T + p.tile - 1) / p.tile;
  const int64_t total = (int64_t)p.Hkv * p.ws.prefix[p.B];
  ui.U = (int64_t)p.Hkv * p.ws.prefix[b] + (int64_t)kvh * ui.nb;
  ui.nseg = 0;
  ui.c0 = 0;
  ui.part = Partition{total > 0 ? total : 1, p.N};
  if (ui.nb > 0 && total > 0) {
    ui.c0 = ui.part.cfirst(ui.U);
    ui.nseg = (int)(ui.part.cfirst(ui.U + ui.nb - 1) - ui.c0 + 1);
    if (ui.nseg > p.R) ui.nseg = p.R;
    if (ui.nseg > kMaxRecords) ui.nseg = kMaxRecords;
  }
  ui.ok = nullptr;
  return ui;
}

__device__ __forceinline__ int64_t slot_of(const ScoreParams &p, int b, int64_t pos) {
  if (p.page_table == nullptr) return (int64_t)b * p.page_size + pos;
  return (int64_t)__ldg(p.page_table + (int64_t)b * p.max_pages + pos / p.page_size) * p.page_size +
         pos % p.page_size;
}

// Block-wide exclusive scan of one int per thread; *total gets the sum.
// sh_warp needs 33 ints.
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
    const int w = lane < nw ? sh_warp[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < nw) sh_warp[lane] = wi - w;
    if (lane == 31) sh_warp[32] = wi;
  }
  __syncthreads();
  const int r = sh_warp[warp] + incl - x;
  *total = sh_warp[32];
  __syncthreads();
  return r;
}

// Over a histogram in shared memory (bin index increasing with score), the
// bin holding the need-th largest element and the count strictly above it.
// Whole block.
__device__ int find_threshold_bin(const uint32_t *hist, int nbins, int need, int *above_out, int *sh_warp,
                                  int *sh_res) {
  const int per = (nbins + blockDim.x - 1) / blockDim.x;
  if (threadIdx.x == 0) {
    sh_res[0] = 0;
    sh_res[1] = 0;
  }
  int cnt = 0;
  for (int k = 0; k < per; ++k) {  // thread i owns the i-th group of bins from the top
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

// Per-head LSE (fp64), max and normaliser of a unit from its segment
// records, as a block-wide reduction: thread t folds the pairs (segment j,
// head h) with h = t % G.
template <int G, int D>
__device__ void unit_lse(const float *rec0, const UnitInfo &ui, float c, double *sh_lse, float *sh_M, float *sh_L,
                         double *sh_red) {
  constexpr int RS = G * (D + 2);
  const int nseg = ui.nseg;
  const int tid = threadIdx.x, nt = blockDim.x, h = tid % G;
  float m = -INFINITY;
  for (int i = tid; i < nseg * G; i += nt)
    if (ui.rec_ok(i / G)) m = fmaxf(m, rec0[(i / G) * RS + h]);
  reinterpret_cast<float *>(sh_red)[tid] = m;
  __syncthreads();
  if (tid < G) {
    float M = -INFINITY;
    for (int t = tid; t < nt; t += G) M = fmaxf(M, reinterpret_cast<float *>(sh_red)[t]);
    sh_M[tid] = M;
  }
  __syncthreads();
  const float M = sh_M[h];
  double L = 0.0;
  for (int i = tid; i < nseg * G; i += nt) {
    const int j = i / G;
    if (!ui.rec_ok(j)) continue;
    const float mj = rec0[j * RS + h];
    if (mj != -INFINITY) L += (double)rec0[j * RS + G + h] * exp((double)c * ((double)mj - (double)M));
  }
  sh_red[tid] = L;
  __syncthreads();
  if (tid < G) {
    double S = 0.0;
    for (int t = tid; t < nt; t += G) S += sh_red[t];
    sh_lse[tid] = (double)c * (double)sh_M[tid] + log(S);
    sh_L[tid] = (float)S;
  }
  __syncthreads();
}


// Exact group score of one position: p_h = 2^(raw_h * a - b_h) with
// a = c log2(e) and b_h = LSE_h log2(e) carried as float pairs, the exponent
// formed with an exact product and a two-sum, so the only rounding of
// consequence is the ex2 approximation (~2^-22 relative); pairwise sum.
__device__ __forceinline__ float exact_score(const float *raw, int G, float c, const double *lse) {
  const double ad = (double)c * kLog2e;
  const float a_hi = (float)ad, a_lo = (float)(ad - (double)a_hi);
  float total = 0.f;
  for (int h0 = 0; h0 < G; h0 += 8) {  // groups of 8 heads, each summed pairwise
    float pr[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int h = h0 + i;
      pr[i] = 0.f;
      if (h >= G) continue;
      const double bd = lse[h] * kLog2e;
      const float b_hi = (float)bd, b_lo = (float)(bd - (double)b_hi);
      const float x = __ldcg(raw + h);
      const float ph = __fmul_rn(x, a_hi);
      const float pl = fmaf(x, a_lo, fmaf(x, a_hi, -ph));  // x*a = ph + pl
      const float sh = __fsub_rn(ph, b_hi);                // two-sum: sh + se = ph - b_hi exactly
      const float z = __fsub_rn(sh, ph);
      const float se = __fadd_rn(__fsub_rn(ph, __fsub_rn(sh, z)), __fsub_rn(-b_hi, z));
      const float yl = (se + pl) - b_lo;
      const float e = ex2_approx(sh);
      pr[i] = fmaf(e, yl * 0.69314718055994531f, e);  // 2^(sh + yl) = 2^sh (1 + yl ln 2)
    }
#pragma unroll
    for (int w = 1; w < 8; w <<= 1)
#pragma unroll
      for (int i = 0; i + w < 8; i += 2 * w) pr[i] += pr[i + w];
    total += pr[0];
  }
  return total >= 0.f ? total : 0.f;  // NaN (bad inputs) ranks lowest
}


// The unit's approximate scores and histogram again, each score scaled by
// 2^E, until the threshold bin is at or above kTrustBin (whole block; runs
// only when the first pass put the k-th score below 2^-96).  Rewrites the
// scores sc[0, nC) and shifts the per-head LSE by E ln 2, so that the filter's
// exact scores carry the same factor.  Returns the threshold bin.
template <int G>
__device__ int rescale_unit(const ScoreParams &p, int nC, const float *lg, float *sc, uint32_t *sh_hist,
                            double *sh_lse, int bin, int *above, int *sh_warp, int *sh_res) {
  const float a = (float)((double)p.c * kLog2e);
  double E = 0.0;
  for (int round = 0; round < 16 && bin < kTrustBin && E < kMaxShift; ++round) {
    const int e_bin = bin >> 4;  // biased fp32 exponent of the threshold bin, 0 when it underflowed
    E += e_bin > 0 ? (double)(kTargetExponent - e_bin) : 200.0;
    if (E > kMaxShift) E = kMaxShift;
    float bh[G];
#pragma unroll
    for (int h = 0; h < G; ++h) bh[h] = (float)(sh_lse[h] * kLog2e - E);
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh_hist[i] = 0u;
    __syncthreads();
    for (int t = threadIdx.x; t < nC; t += blockDim.x) {
      float pr[G];
#pragma unroll
      for (int h = 0; h < G; ++h) pr[h] = ex2_approx(fmaf(__ldcg(lg + (size_t)t * G + h), a, -bh[h]));
#pragma unroll
      for (int w = 1; w < G; w <<= 1)
#pragma unroll
        for (int h = 0; h + w < G; h += 2 * w) pr[h] += pr[h + w];
      const float sv = pr[0] >= 0.f ? pr[0] : 0.f;
      sc[t] = sv;
      atomicAdd(&sh_hist[__float_as_uint(sv) >> kHistShift], 1u);
    }
    __syncthreads();
    bin = find_threshold_bin(sh_hist, kHistBins, p.k_global, above, sh_warp, sh_res);
  }
  if (threadIdx.x < G) sh_lse[threadIdx.x] -= E * kLn2;
  __syncthreads();
  return bin;
}

// One combine CTA of unit u: out = sum_j o_j exp(c (m_j - M_h)) / L_h over
// output elements [comb * kCombineElems, ...), the records' (m, l, o) from the
// attention pass (sh_M, sh_L: the unit's per-head max and normaliser; the
// histogram's shared memory holds the weights).
template <int G, int D>
__device__ void combine_unit(const ScoreParams &p, const UnitInfo &ui, int64_t u, int comb, const float *sh_M,
                             const float *sh_L, uint32_t *sh_hist) {
  constexpr int RS = G * (D + 2);
  const int b = (int)(u / p.Hkv), kvh = (int)(u % p.Hkv);
  const float *rec0 = p.ws.records + (size_t)u * p.R * RS;
  const int e0 = comb * kCombineElems, e1 = min(G * D, e0 + kCombineElems);
  const int h0 = e0 / D, nh = e1 > e0 ? (e1 - 1) / D - h0 + 1 : 0;
  // the weights exp(c (m_j - M_h)) / L_h of this CTA's heads, once per (record, head)
  float *wts = reinterpret_cast<float *>(sh_hist);  // [nseg][nh] (nseg * nh <= kHistBins)
  for (int i = threadIdx.x; i < ui.nseg * nh; i += blockDim.x) {
    const int j = i / nh, h = h0 + i % nh;
    const float mj = ui.rec_ok(j) ? rec0[j * RS + h] : -INFINITY;
    wts[i] = mj != -INFINITY && sh_L[h] > 0.f ? expf(p.c * (mj - sh_M[h])) / sh_L[h] : 0.f;
  }
  __syncthreads();
  const int64_t ob = ((int64_t)b * p.Hkv * G + (int64_t)kvh * G) * D;
  for (int e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const int hi = e / D - h0;
    float acc = 0.f;
#pragma unroll 8
    for (int j = 0; j < ui.nseg; ++j) {
      const float w = wts[j * nh + hi];
      if (w != 0.f) acc += rec0[j * RS + 2 * G + e] * w;
    }
    if (p.out_dtype == 0) static_cast<float *>(p.out)[ob + e] = acc;
    else static_cast<__nv_bfloat16 *>(p.out)[ob + e] = __float2bfloat16_rn(acc);
  }
}

}  // namespace

}  // namespace hs2
