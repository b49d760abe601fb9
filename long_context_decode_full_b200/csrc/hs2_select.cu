// hs2_select.cu -- token-level selection of a Hybrid Block (HySparse2
// announcement: the full layer picks important positions from its attention
// scores; selection is per token; the most recent `window` tokens are always
// kept plus the top `k_global` tokens from outside that window).
//
// Score of position t for KV head j: sum over the query heads h of j's GQA
// group of the softmax probability p_{h,t} = exp(c * s_{h,t} - LSE_h).
//
// Three kernels on the CUDA cores:
//   score  -- grid (chunk, kv head, sequence) + combine CTAs per unit; a
//             chunk (2048..65536 positions) is sized per call so the grid is
//             one wave.  Score CTAs rebuild each head's LSE from the segment
//             records (a parallel fp64 reduction), then turn the raw logits of
//             their chunk into approximate group scores (one FMA and one ex2
//             per head, relative error below 1e-5) and a 4096-bin histogram of
//             their top bits (16 bins per octave); the last chunk to finish
//             (atomic ticket, no waiting) finds the bin b holding the
//             k_global-th largest approximate score.  The combine CTAs merge
//             the records into the attention output.
//   filter -- each warp owns one or two 512-position sub-ranges and writes,
//             in position order, the positions whose approximate score is
//             above bin b widened by a 4e-4 margin (certainly above the k-th
//             exact score) and, with exact scores (exponent formed in
//             float-float, so only ex2's own rounding is left), the positions
//             inside that widened bin: the guard band that holds every
//             position the exact k-th score can hinge on.
//   final  -- one CTA per unit: the need-th best guard-band entry by exact
//             score, ties to the lower position (the lists are
//             position-ordered), found by direct ranks for bands up to 768
//             entries and by a radix select otherwise, then a merge of the two
//             sorted lists and the forced window into the index list.
// Scores are >= 0, so their IEEE bit patterns order like the values.
#include "hs2_internal.h"
#include "hs2_select_common.cuh"

namespace hs2 {

namespace {

// ------------------------------------------------------------------ score
// Positions per thread and batch (two batches in flight): 16 logits per batch.
template <int G>
constexpr int score_loads() { return G >= 16 ? 1 : 16 / G; }

// Loads the logits of positions tb + q * kScoreThreads (q < score_loads) below t1.
template <int G>
__device__ __forceinline__ void load_logits(float (&raw)[score_loads<G>()][G], const float *lg, int tb, int t1) {
  constexpr int kScoreLoads = score_loads<G>();
#pragma unroll
  for (int q = 0; q < kScoreLoads; ++q) {
    const int t = tb + q * kScoreThreads;
    if (t >= t1) {
#pragma unroll
      for (int h = 0; h < G; ++h) raw[q][h] = 0.f;
      continue;
    }
    if constexpr (G % 4 == 0) {
#pragma unroll
      for (int h4 = 0; h4 < G / 4; ++h4) {
        const float4 v4 = __ldcs(reinterpret_cast<const float4 *>(lg + (size_t)t * G) + h4);
        raw[q][4 * h4] = v4.x;
        raw[q][4 * h4 + 1] = v4.y;
        raw[q][4 * h4 + 2] = v4.z;
        raw[q][4 * h4 + 3] = v4.w;
      }
    } else {
#pragma unroll
      for (int h = 0; h < G; ++h) raw[q][h] = __ldcs(lg + (size_t)t * G + h);
    }
  }
}

template <int G, int D>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(const ScoreParams p) {
  __shared__ uint32_t sh_hist[kHistBins];
  __shared__ double sh_red[kScoreThreads];
  __shared__ double sh_lse[G];
  __shared__ float sh_M[G], sh_L[G];
  __shared__ int sh_warp[33], sh_res[2], sh_last;
  __shared__ uint8_t sh_ok[kMaxRecords];
  constexpr int RS = G * (D + 2);
  griddep_wait();
  griddep_launch_dependents();
  const int chunk = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  // the last p.ncomb x-indices are the unit's combine CTAs, kCombineElems
  // output elements each
  const int comb = chunk - ((int)gridDim.x - p.ncomb);
  const bool combine = comb >= 0;
  UnitInfo ui = unit_info(p, b, kvh);
  const int n_chunks = ui.select ? (ui.nC + p.score_chunk - 1) / p.score_chunk : 0;
  if (!combine && chunk >= n_chunks) return;
  const int64_t u = (int64_t)b * p.Hkv + kvh;
  const int t0 = chunk * p.score_chunk, t1 = min(ui.nC, t0 + p.score_chunk);
  const float *lg = p.ws.logits + (size_t)u * p.ustride * G;
  // the LSE first: its dependent record loads would otherwise queue behind
  // every CTA's first batch of logits
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sh_hist[i] = 0u;
  mark_records(ui, sh_ok);
  const float *rec0 = p.ws.records + (size_t)u * p.R * RS;
  unit_lse<G, D>(rec0, ui, p.c, sh_lse, sh_M, sh_L, sh_red);
  constexpr int kScoreLoads = score_loads<G>();
  float raw[kScoreLoads][G], raw2[kScoreLoads][G];
  if (!combine) load_logits<G>(raw, lg, t0 + threadIdx.x, t1);

  if (combine) {
    combine_unit<G, D>(p, ui, u, comb, sh_M, sh_L, sh_hist);
    return;
  }

  float *sc = p.ws.scores + (size_t)u * p.ustride;
  // approximate p_h = 2^(raw * a - b_h), a = c log2(e), b_h = LSE_h log2(e):
  // the exponent rounds once in fp32 (|x| < 64: absolute error < 4e-6), so
  // the score is within ~1e-5 relative -- only used to bin positions
  const float a = (float)((double)p.c * kLog2e);
  float bh[G];
#pragma unroll
  for (int h = 0; h < G; ++h) bh[h] = (float)(sh_lse[h] * kLog2e);
  constexpr int kStep = kScoreLoads * kScoreThreads;
  auto score_batch = [&](const float (&r)[kScoreLoads][G], int tb) {
#pragma unroll
    for (int q = 0; q < kScoreLoads; ++q) {
      const int t = tb + q * kScoreThreads;
      if (t >= t1) break;
      float pr[G];
#pragma unroll
      for (int h = 0; h < G; ++h) pr[h] = ex2_approx(fmaf(r[q][h], a, -bh[h]));
#pragma unroll
      for (int w = 1; w < G; w <<= 1)  // pairwise sum of the group's probabilities
#pragma unroll
        for (int h = 0; h + w < G; h += 2 * w) pr[h] += pr[h + w];
      const float s = pr[0] >= 0.f ? pr[0] : 0.f;  // NaN (bad inputs) ranks lowest
      sc[t] = s;
      atomicAdd(&sh_hist[__float_as_uint(s) >> kHistShift], 1u);
    }
  };
  // two batches in flight: the next one loads while the current one is scored
  // (the first batch was loaded before the LSE)
  for (int tb = t0 + threadIdx.x; tb < t1; tb += 2 * kStep) {
    load_logits<G>(raw2, lg, tb + kStep, t1);
    score_batch(raw, tb);
    load_logits<G>(raw, lg, tb + 2 * kStep, t1);
    score_batch(raw2, tb + kStep);
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
  int bin = find_threshold_bin(sh_hist, kHistBins, p.k_global, &above, sh_warp, sh_res);
  if (bin < kTrustBin) bin = rescale_unit<G>(p, ui.nC, lg, sc, sh_hist, sh_lse, bin, &above, sh_warp, sh_res);
  if (threadIdx.x == 0) p.ws.thr[u] = make_int2(bin, above);
  if (threadIdx.x < G) p.ws.lse[u * kMaxGroup + threadIdx.x] = sh_lse[threadIdx.x];
}

// ------------------------------------------------------------------ filter
constexpr int kFilterRounds = kSubRange / 128;
constexpr int kFilterSubsMax = 2;  // sub-ranges per warp (p.filter_subs <= this)

// Lane l of round r holds positions s0 + 128 r + 4 l .. +3 (one float4) of
// sub-range `sub`, so (round, lane, element) order is position order.
__device__ __forceinline__ void load_sub_scores(const float *sc, int sub, int nC, float4 (&v)[kFilterRounds]) {
  const int lane = threadIdx.x & 31;
  const int s0 = sub * kSubRange, s1 = min(nC, s0 + kSubRange);
#pragma unroll
  for (int r = 0; r < kFilterRounds; ++r) {
    const int t = s0 + 128 * r + 4 * lane;
    v[r] = t + 3 < s1 ? __ldcs(reinterpret_cast<const float4 *>(sc + t))
                      : make_float4(t < s1 ? sc[t] : 0.f, t + 1 < s1 ? sc[t + 1] : 0.f,
                                    t + 2 < s1 ? sc[t + 2] : 0.f, 0.f);
  }
}

// One warp, one 512-position sub-range: writes, in position order, the
// positions certainly above the k-th exact score and the guard band (with
// exact scores), and the two counts.
__device__ void filter_sub(const ScoreParams &p, int64_t u, int sub, int nC, float lo, float hi,
                           const float4 (&v)[kFilterRounds], int *band, const double *lse) {
  const int lane = threadIdx.x & 31;
  const int s0 = sub * kSubRange, s1 = min(nC, s0 + kSubRange);
  int32_t *above = p.ws.above + (size_t)u * p.ustride + s0;
  uint2 *eqs = p.ws.cand + (size_t)u * p.ustride + s0;
  int na = 0, ne = 0;
#pragma unroll
  for (int r = 0; r < kFilterRounds; ++r) {
    const int t = s0 + 128 * r + 4 * lane;
    const float f[4] = {v[r].x, v[r].y, v[r].z, v[r].w};
    int ca = 0, ce = 0;
    bool a[4], e[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const bool valid = t + k < s1;
      a[k] = valid && f[k] >= hi;               // certainly above the k-th exact score
      e[k] = valid && f[k] >= lo && f[k] < hi;  // guard band
      ca += a[k];
      ce += e[k];
    }
    // warp exclusive scans of the per-lane counts
    int xa = ca, xe = ce;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, xa, o), ye = __shfl_up_sync(0xffffffffu, xe, o);
      if (lane >= o) {
        xa += ya;
        xe += ye;
      }
    }
    const int ta = __shfl_sync(0xffffffffu, xa, 31), te = __shfl_sync(0xffffffffu, xe, 31);
    int oa = na + xa - ca, oe = ne + xe - ce;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (a[k]) above[oa++] = t + k;
      if (e[k]) band[oe++] = t + k;
    }
    na += ta;
    ne += te;
  }
  // guard band: exact scores, the whole warp working through the list with
  // every load in flight together
  __syncwarp();
  for (int i = lane; i < ne; i += 32) {
    const int pos = band[i];
    const float ex = exact_score(p.ws.logits + ((size_t)u * p.ustride + pos) * p.G, p.G, p.c, lse);
    eqs[i] = make_uint2(__float_as_uint(ex), (uint32_t)pos);
  }
  __syncwarp();
  if (lane == 0) p.ws.subcnt[(size_t)u * p.nsub + sub] = make_int2(na, ne);
}

// Each warp owns p.filter_subs sub-ranges (strided by the CTA's warps), with
// the scores of all of them loaded up front.
__global__ void __launch_bounds__(kScoreThreads) filter_kernel(const ScoreParams p) {
  __shared__ int sh_band[kScoreThreads / 32][kSubRange];  // each warp's guard-band positions
  griddep_wait();
  griddep_launch_dependents();
  const int chunk = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int T = clamp_len(__ldg(p.seq_lens + b), (int)p.t_cap);
  const int nC = max(0, T - p.window);
  const int fchunk = kSubRange * (kScoreThreads / 32) * p.filter_subs;  // positions per CTA
  if (nC <= p.k_global || p.k_global == 0 || chunk * fchunk >= nC) return;
  const int64_t u = (int64_t)b * p.Hkv + kvh;
  const int warp = threadIdx.x >> 5;
  constexpr int kWarps = kScoreThreads / 32;
  const float *sc = p.ws.scores + (size_t)u * p.ustride;
  const int sub0 = chunk * (fchunk / kSubRange) + warp;
  float4 v[kFilterSubsMax][kFilterRounds];
#pragma unroll
  for (int k = 0; k < kFilterSubsMax; ++k)
    if (k < p.filter_subs && (sub0 + k * kWarps) * kSubRange < nC) load_sub_scores(sc, sub0 + k * kWarps, nC, v[k]);
  // The k-th exact score lies in the threshold bin [lo, hi) widened by the
  // approximation error (< 2e-5 relative even for logits of several hundred);
  // the band keeps a 4e-4 margin on both sides.
  const int bin1 = p.ws.thr[u].x;
  const float lo = __uint_as_float((uint32_t)bin1 << kHistShift) * (1.f - kBandMargin);
  const float hi = bin1 >= 0xFEF ? INFINITY : __uint_as_float((uint32_t)(bin1 + 1) << kHistShift) * (1.f + kBandMargin);
  __shared__ double lse[kMaxGroup];
  if (threadIdx.x < p.G) lse[threadIdx.x] = p.ws.lse[u * kMaxGroup + threadIdx.x];
  __syncthreads();
#pragma unroll
  for (int k = 0; k < kFilterSubsMax; ++k) {
    const int sub = sub0 + k * kWarps;
    if (k >= p.filter_subs || sub * kSubRange >= nC) break;
    filter_sub(p, u, sub, nC, lo, hi, v[k], sh_band[warp], lse);
  }
}

// ------------------------------------------------------------------ final
// Block-wide exclusive scan of two ints per thread at once.  sh needs 66 ints.
__device__ __forceinline__ int2 block_exclusive_scan2(int2 x, int *sh, int2 *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  int ia = x.x, ie = x.y;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int ya = __shfl_up_sync(0xffffffffu, ia, o), ye = __shfl_up_sync(0xffffffffu, ie, o);
    if (lane >= o) {
      ia += ya;
      ie += ye;
    }
  }
  if (lane == 31) {
    sh[warp] = ia;
    sh[33 + warp] = ie;
  }
  __syncthreads();
  if (warp == 0) {
    const int wa = lane < nw ? sh[lane] : 0, we = lane < nw ? sh[33 + lane] : 0;
    int sa = wa, se = we;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, sa, o), ye = __shfl_up_sync(0xffffffffu, se, o);
      if (lane >= o) {
        sa += ya;
        se += ye;
      }
    }
    if (lane < nw) {
      sh[lane] = sa - wa;
      sh[33 + lane] = se - we;
    }
    if (lane == 31) {
      sh[32] = sa;
      sh[65] = se;
    }
  }
  __syncthreads();
  const int2 r = make_int2(sh[warp] + ia - x.x, sh[33 + warp] + ie - x.y);
  *total = make_int2(sh[32], sh[65]);
  __syncthreads();
  return r;
}

// Exclusive offsets of the per-sub-range counts (above, in-bin) into shared
// memory; off_x[nsub] holds the totals.
__device__ void scan_subcounts(const int2 *cnt, int nsub, int *off_a, int *off_e, int *sh_scan) {
  int carry_a = 0, carry_e = 0;
  for (int base = 0; base < nsub; base += blockDim.x) {
    const int s = base + threadIdx.x;
    const int2 c = s < nsub ? __ldcg(cnt + s) : make_int2(0, 0);
    int2 tot;
    const int2 x = block_exclusive_scan2(c, sh_scan, &tot);
    if (s < nsub) {
      off_a[s] = carry_a + x.x;
      off_e[s] = carry_e + x.y;
    }
    carry_a += tot.x;
    carry_e += tot.y;
  }
  if (threadIdx.x == 0) {
    off_a[nsub] = carry_a;
    off_e[nsub] = carry_e;
  }
  __syncthreads();
}

// sub-range holding list element i (off ascending over [0, n], off[n] = total)
__device__ __forceinline__ int find_sub(const int *off, int n, int i) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Guard bands up to this size are ranked directly (each element against all
// others, shared-memory broadcasts); larger ones take the radix select.
constexpr int kRankSelectMax = 768;
constexpr int kPerThread = kMaxSelect / kFinalThreads;  // list entries per thread, at most

__global__ void __launch_bounds__(kFinalThreads) final_kernel(const ScoreParams p) {
  extern __shared__ int fsm[];  // off_a[nsub+1], off_e[nsub+1], list_a[kMaxSelect], list_c[kMaxSelect],
                                // slot_c[kMaxSelect], then the in-bin list (bits, position) when it
                                // fits: list_e[kMaxSelect]
  __shared__ uint32_t sh_hist[2048];
  __shared__ int sh_warp[66], sh_res[2], sh_ties;
  griddep_wait();
  griddep_launch_dependents();
  const int kvh = blockIdx.x, b = blockIdx.y;
  const int T = clamp_len(__ldg(p.seq_lens + b), (int)p.t_cap);
  const int nC = max(0, T - p.window);
  const int L = p.window + p.k_global;
  const int64_t u = (int64_t)b * p.Hkv + kvh;
  int32_t *idx = p.idx_out + (size_t)u * L;
  const bool select = nC > p.k_global && p.k_global > 0;
  int *off_a = fsm, *off_e = fsm + p.nsub + 1;
  int *list_a = fsm + 2 * (p.nsub + 1), *list_c = list_a + kMaxSelect, *slot_c = list_c + kMaxSelect;
  uint2 *list_e = reinterpret_cast<uint2 *>(slot_c + kMaxSelect);
  // the forced window's slots, looked up now and written last
  int sw[kPerThread];
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int t = nC + threadIdx.x + k * kFinalThreads;
    sw[k] = t < T ? (int)slot_of(p, b, t) : -1;
  }

  int n_sel = 0;  // selectable positions kept (all before the window)
  if (select) {
    const int nsub = (nC + kSubRange - 1) / kSubRange;
    scan_subcounts(p.ws.subcnt + (size_t)u * p.nsub, nsub, off_a, off_e, sh_warp);
    const int A = min(off_a[nsub], kMaxSelect), E = off_e[nsub];
    const int32_t *above = p.ws.above + (size_t)u * p.ustride;
    const uint2 *eqs_g = p.ws.cand + (size_t)u * p.ustride;
    // the above-threshold positions (fewer than k_global), already in order,
    // and the in-bin list when it fits, in one round of loads
    const bool e_in_smem = E <= kMaxSelect;
    const bool rank_path = E <= kRankSelectMax;
    for (int i = threadIdx.x; i < A; i += blockDim.x) {
      const int s = find_sub(off_a, nsub, i);
      list_a[i] = __ldcg(above + (size_t)s * kSubRange + (i - off_a[s]));
    }
    if (e_in_smem)
      for (int i = threadIdx.x; i < E; i += blockDim.x) {
        const int s = find_sub(off_e, nsub, i);
        list_e[i] = __ldcg(eqs_g + (size_t)s * kSubRange + (i - off_e[s]));
      }
    __syncthreads();
    // output slots of the above list and of the guard band, in flight during the selection
    int sa[kPerThread], se[2];
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int i = threadIdx.x + k * kFinalThreads;
      sa[k] = i < A ? (int)slot_of(p, b, list_a[i]) : -1;
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int i = threadIdx.x + k * kFinalThreads;
      se[k] = rank_path && i < E ? (int)slot_of(p, b, (int)list_e[i].y) : -1;
    }
    const int need = p.k_global - A;  // band elements to keep
    int taken = 0;
    if (rank_path) {
      // element i (position order) is kept when fewer than `need` elements
      // outrank it: a higher exact score, or an equal one at a lower position
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int i = threadIdx.x + k * kFinalThreads;
        int take = 0;
        if (i < E) {
          const uint32_t si = list_e[i].x;
          int r = 0;
#pragma unroll 4
          for (int j = 0; j < E; ++j) {
            const uint32_t sj = list_e[j].x;
            r += (sj > si) | ((sj == si) & (j < i));
          }
          take = r < need ? 1 : 0;
        }
        int tot;
        const int pos = taken + block_exclusive_scan(take, sh_warp, &tot);
        if (take) {
          list_c[pos] = (int)list_e[i].y;
          slot_c[pos] = se[k];
        }
        taken += tot;
      }
    } else {
      auto in_bin = [&](int i) -> uint2 {  // i-th guard-band element in position order
        if (e_in_smem) return list_e[i];
        const int s = find_sub(off_e, nsub, i);
        return __ldcg(eqs_g + (size_t)s * kSubRange + (i - off_e[s]));
      };
      // radix select of the need-th largest exact score: bits 31..21, 20..10, 9..0
      int rem = need;
      uint32_t prefix = 0u, mask = 0u;
      const int shifts[3] = {21, 10, 0}, widths[3] = {11, 11, 10};
      for (int round = 0; round < 3; ++round) {
        const int sh = shifts[round], nb = 1 << widths[round];
        for (int i = threadIdx.x; i < nb; i += blockDim.x) sh_hist[i] = 0u;
        __syncthreads();
        for (int i = threadIdx.x; i < E; i += blockDim.x) {
          const uint32_t bits = in_bin(i).x;
          if ((bits & mask) == prefix) atomicAdd(&sh_hist[(bits >> sh) & (nb - 1)], 1u);
        }
        __syncthreads();
        int ab;
        const int bin = find_threshold_bin(sh_hist, nb, rem, &ab, sh_warp, sh_res);
        rem -= ab;
        prefix |= (uint32_t)bin << sh;
        mask |= (uint32_t)(nb - 1) << sh;
        if (round == 2 && threadIdx.x == 0) sh_ties = (int)sh_hist[bin];  // elements equal to the k-th score
      }
      __syncthreads();
      const uint32_t kth = prefix;  // the exact k_global-th score; `rem` of its ties are kept
      const bool keep_all_ties = sh_ties <= rem;
      // walk the in-bin list in position order: keep scores above kth and the
      // first `rem` equal to it
      int ties = 0;
      for (int base = 0; base < E; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const uint2 cv = i < E ? in_bin(i) : make_uint2(0u, 0u);
        int take;
        if (keep_all_ties) {
          take = (i < E && cv.x >= kth) ? 1 : 0;
        } else {
          const int is_tie = (i < E && cv.x == kth) ? 1 : 0;
          int tie_tot;
          const int tie_rank = ties + block_exclusive_scan(is_tie, sh_warp, &tie_tot);
          take = (i < E && (cv.x > kth || (is_tie && tie_rank < rem))) ? 1 : 0;
          ties += tie_tot;
        }
        int take_tot;
        const int pos = taken + block_exclusive_scan(take, sh_warp, &take_tot);
        if (take && pos < kMaxSelect) {
          list_c[pos] = (int)cv.y;
          slot_c[pos] = (int)slot_of(p, b, cv.y);
        }
        taken += take_tot;
      }
    }
    __syncthreads();
    // merge two position-ordered lists: rank = own index + smaller elements of the other list
    const int nc = min(taken, kMaxSelect);
    n_sel = A + nc;
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int i = threadIdx.x + k * kFinalThreads;
      if (i >= A) break;
      const int v = list_a[i];
      int lo = 0, hi = nc;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (list_c[mid] < v) lo = mid + 1; else hi = mid;
      }
      if (i + lo < L) idx[i + lo] = sa[k];
    }
    for (int i = threadIdx.x; i < nc; i += blockDim.x) {
      const int v = list_c[i];
      int lo = 0, hi = A;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (list_a[mid] < v) lo = mid + 1; else hi = mid;
      }
      if (i + lo < L) idx[i + lo] = slot_c[i];
    }
  } else if (p.k_global > 0) {  // every selectable position is kept
    n_sel = nC;
    for (int t = threadIdx.x; t < nC && t < L; t += blockDim.x) idx[t] = (int32_t)slot_of(p, b, t);
  }
  // the forced window follows every selectable position
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int t = nC + threadIdx.x + k * kFinalThreads;
    const int o = n_sel + (t - nC);
    if (t < T && o < L) idx[o] = sw[k];
  }
  const int n_total = n_sel + (T - nC);
  for (int i = n_total + threadIdx.x; i < L; i += blockDim.x) idx[i] = -1;
}

template <int G>
cudaError_t launch_score_g(const ScoreParams &p, dim3 grid, cudaStream_t s) {
  if (p.D == 64) return launch_ex(score_kernel<G, 64>, grid, dim3(kScoreThreads), 0, s, 0, p);
  return launch_ex(score_kernel<G, 128>, grid, dim3(kScoreThreads), 0, s, 0, p);
}

size_t final_smem_bytes(int nsub) { return (size_t)(2 * (nsub + 1) + 5 * kMaxSelect) * sizeof(int); }

}  // namespace

cudaError_t launch_select(const ScoreParams &p, cudaStream_t s) {
  const int chunks = (int)((p.t_cap + p.score_chunk - 1) / p.score_chunk);
  cudaError_t e;
  const dim3 sgrid(chunks + p.ncomb, p.Hkv, p.B);  // + the combine CTAs of each unit
  switch (p.G) {
    case 1: e = launch_score_g<1>(p, sgrid, s); break;
    case 2: e = launch_score_g<2>(p, sgrid, s); break;
    case 4: e = launch_score_g<4>(p, sgrid, s); break;
    case 8: e = launch_score_g<8>(p, sgrid, s); break;
    case 16: e = launch_score_g<16>(p, sgrid, s); break;
    case 32: e = launch_score_g<32>(p, sgrid, s); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return launch_select_after_score(p, s);
}

cudaError_t launch_select_after_score(const ScoreParams &p, cudaStream_t s) {
  const int fchunk = kSubRange * (kScoreThreads / 32) * p.filter_subs;
  const int fchunks = (int)((p.t_cap + fchunk - 1) / fchunk);
  cudaError_t e = launch_ex(filter_kernel, dim3(fchunks, p.Hkv, p.B), dim3(kScoreThreads), 0, s, 0, p);
  if (e != cudaSuccess) return e;
  const size_t smem = final_smem_bytes(p.nsub);
  e = set_smem_once(reinterpret_cast<const void *>(final_kernel), (int)smem);
  if (e != cudaSuccess) return e;
  return launch_ex(final_kernel, dim3(p.Hkv, p.B), dim3(kFinalThreads), smem, s, 0, p);
}

}  // namespace hs2
