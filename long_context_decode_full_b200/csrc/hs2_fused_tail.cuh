// hs2_fused_tail.cuh -- the score pass run inside the persistent attention
// kernel (the fused full-attention + selection call).  HySparse2 announcement,
// "KV Reuse" section: the full layer picks the positions the sparse layers
// will read while finishing its own computation.
//
// After its last tile a CTA waits at a grid barrier (every segment record and
// logit of the call is written then), and scores the positions it attended
// itself: for each unit its tile range touches, the unit's per-head LSE from
// the segment records, the approximate group scores of those positions with
// their logits still in L2 (several loads in flight per thread), and the
// unit's 4096-bin histogram.  The CTA that completes a unit's histogram
// (ticket, no waiting) finds its threshold bin -- with the common 2^E factor
// when the k-th score lies below fp32's range -- and the unit's first CTA
// writes the attention output from the records.  The filter and final kernels
// follow as separate launches, exactly as after the score kernel.
//
// The grid barrier needs every CTA resident at once: the kernel is launched
// cooperatively (one CTA per SM).  Its wait is bounded; on expiry the CTA sets
// the workspace's sticky flag and skips the score pass.
#pragma once

#include "hs2_internal.h"
#include "hs2_select_common.cuh"

namespace hs2 {

namespace {

constexpr uint32_t kErrGridWait = 8u;  // a CTA gave up at the fused call's grid barrier

// The score pass streams each segment's logits into the idle K/V stages with
// untiled bulk copies of kTailChunk bytes, up to kTailBufs of them in flight.
constexpr int kTailChunk = 16384;
constexpr int kTailBufs = 12;

// Shared-memory arrays of the score pass (overlaid on the idle K/V stages,
// the copy buffers after them).
struct TailSmem {
  uint64_t bars[kTailBufs];
  uint32_t hist[kHistBins];
  double red[512];
  double lse[kMaxGroup];
  float M[kMaxGroup], L[kMaxGroup];
  int warp[33], res[2], last, ok_flag;
  uint8_t ok[kMaxRecords];
};
constexpr size_t kTailBufOffset = (sizeof(TailSmem) + 1023) / 1024 * 1024;

// Copy-buffer state of the score pass, uniform over the block: chunks are
// issued and consumed in one global order, chunk q in buffer q % nbuf.
struct TailStream {
  uint32_t buf0;  // shared address of buffer 0
  int nbuf;
  uint32_t issued, consumed;
};

// Grid-wide barrier over `nblocks` co-resident CTAs.  `count` is zero between
// calls (the last arriver returns it to zero before it releases the others by
// bumping `gen`); the wait gives up after `limit` clock cycles.  Whole block.
__device__ bool grid_barrier(uint32_t *count, uint32_t *gen, uint32_t nblocks, int *flag,
                             long long limit = kSpinLimitCycles) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's records, logits and counters before its arrival
    const uint32_t g0 = *reinterpret_cast<volatile uint32_t *>(gen);  // read before arriving
    bool ok = true;
    if (atomicAdd(count, 1u) == nblocks - 1) {
      atomicExch(count, 0u);
      __threadfence();
      atomicAdd(gen, 1u);
    } else {
      const long long t0 = clock64();
      while (*reinterpret_cast<volatile uint32_t *>(gen) == g0) {
        if (clock64() - t0 > limit) {
          ok = false;
          break;
        }
        __nanosleep(100);
      }
    }
    __threadfence();
    *flag = ok ? 1 : 0;
  }
  __syncthreads();
  return *flag != 0;
}

// Issues the first copies of positions [t0, t1) of one unit (thread 0; the
// block's counters advance alike).  Returns the chunks of the range.
template <int G>
__device__ int tail_issue_first(const float *lg, int t0, int t1, TailSmem *ts, TailStream &st) {
  constexpr int PPC = kTailChunk / (G * 4);  // positions per chunk
  const int nchunks = (t1 - t0 + PPC - 1) / PPC;
  const int first = min(st.nbuf, nchunks);
  for (int k = 0; k < first; ++k) {
    if (threadIdx.x == 0) {
      const int tp = t0 + k * PPC, n = min(PPC, t1 - tp);
      const uint32_t bytes = ((uint32_t)n * G * 4 + 15u) & ~15u;  // stays inside the unit's logit rows
      const int buf = (int)(st.issued % (uint32_t)st.nbuf);
      fence_proxy_async_smem();  // the buffer's earlier reads come first
      mbar_arrive_expect_tx(&ts->bars[buf], bytes);
      bulk_load(st.buf0 + (uint32_t)buf * kTailChunk, lg + (size_t)tp * G, bytes, &ts->bars[buf]);
    }
    ++st.issued;
  }
  return nchunks;
}

// Approximate group scores of positions [t0, t1) of one unit (the same
// arithmetic as the score kernel) into sc[] and the shared histogram.  The
// logits arrive in kTailChunk-byte bulk copies (the first ones issued by
// tail_issue_first); thread 0 keeps up to nbuf in flight.  Each thread scores
// KP positions per round, loads first, so their exponentials overlap.
// Returns false (uniformly) when a copy did not land in time.
template <int G>
__device__ bool tail_score_range(const float *lg, float *sc, int t0, int t1, int nchunks, float c,
                                 const double *lse, TailSmem *ts, TailStream &st) {
  constexpr int PPC = kTailChunk / (G * 4);
  constexpr int KP = G >= 32 ? 1 : (G >= 8 ? 32 / G : 8);  // positions per thread and round
  const int nthr = blockDim.x, tid = threadIdx.x;
  const float a = (float)((double)c * kLog2e);
  float bh[G];
#pragma unroll
  for (int h = 0; h < G; ++h) bh[h] = (float)(lse[h] * kLog2e);
  bool ok = true;
  for (int k = 0; k < nchunks; ++k) {
    const int buf = (int)(st.consumed % (uint32_t)st.nbuf);
    const uint32_t parity = (st.consumed / (uint32_t)st.nbuf) & 1u;
    ++st.consumed;
    ok = __syncthreads_and(ok && mbar_wait(&ts->bars[buf], parity)) != 0;
    if (!ok) {  // give the copies still in flight a bounded time to land before the CTA exits
      if (tid == 0)
        for (uint32_t q = st.consumed - 1u; q < st.issued; ++q)
          mbar_wait(&ts->bars[q % (uint32_t)st.nbuf], (q / (uint32_t)st.nbuf) & 1u, 40000000LL);
      __syncthreads();
      break;
    }
    const float *src = reinterpret_cast<const float *>(reinterpret_cast<const uint8_t *>(ts) + kTailBufOffset +
                                                       (size_t)buf * kTailChunk);
    const int tp = t0 + k * PPC, n = min(PPC, t1 - tp);
    for (int base = 0; base < n; base += KP * nthr) {
      float v[KP][G];
#pragma unroll
      for (int q = 0; q < KP; ++q) {
        const int i = base + tid + q * nthr;
        if constexpr (G % 4 == 0) {
#pragma unroll
          for (int h4 = 0; h4 < G / 4; ++h4) {
            const float4 v4 = i < n ? reinterpret_cast<const float4 *>(src + i * G)[h4] : make_float4(0, 0, 0, 0);
            v[q][4 * h4] = v4.x;
            v[q][4 * h4 + 1] = v4.y;
            v[q][4 * h4 + 2] = v4.z;
            v[q][4 * h4 + 3] = v4.w;
          }
        } else {
#pragma unroll
          for (int h = 0; h < G; ++h) v[q][h] = i < n ? src[i * G + h] : 0.f;
        }
      }
      float sv[KP];
#pragma unroll
      for (int q = 0; q < KP; ++q) {
        float pr[G];
#pragma unroll
        for (int h = 0; h < G; ++h) pr[h] = ex2_approx(fmaf(v[q][h], a, -bh[h]));
#pragma unroll
        for (int w = 1; w < G; w <<= 1)
#pragma unroll
          for (int h = 0; h + w < G; h += 2 * w) pr[h] += pr[h + w];
        sv[q] = pr[0] >= 0.f ? pr[0] : 0.f;  // NaN (bad inputs) ranks lowest
      }
#pragma unroll
      for (int q = 0; q < KP; ++q) {
        const int i = base + tid + q * nthr;
        if (i < n) {
          sc[tp + i] = sv[q];
          atomicAdd(&ts->hist[__float_as_uint(sv[q]) >> kHistShift], 1u);
        }
      }
    }
    __syncthreads();  // the buffer is read
    if (k + st.nbuf < nchunks) {
      if (tid == 0) {
        const int kk = k + st.nbuf;
        const int tq = t0 + kk * PPC, nq = min(PPC, t1 - tq);
        const uint32_t bytes = ((uint32_t)nq * G * 4 + 15u) & ~15u;
        const int b2 = (int)(st.issued % (uint32_t)st.nbuf);
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&ts->bars[b2], bytes);
        bulk_load(st.buf0 + (uint32_t)b2 * kTailChunk, lg + (size_t)tq * G, bytes, &ts->bars[b2]);
      }
      ++st.issued;
    }
  }
  return ok;
}

// The score pass of this CTA over linear tiles [g0, g1), then its share of
// the attention outputs (whole block).  ring_bytes: shared memory available
// from ts on (the K/V stages).
template <int G, int D>
__device__ void fused_tail(const ScoreParams &sp, int64_t g0, int64_t g1, TailSmem *ts, size_t ring_bytes) {
  constexpr int RS = G * (D + 2);
  TailStream st;
  st.buf0 = smem_u32(ts) + (uint32_t)kTailBufOffset;
  st.nbuf = min(kTailBufs, (int)((ring_bytes - kTailBufOffset) / kTailChunk));
  st.issued = st.consumed = 0u;
  if (threadIdx.x == 0) {
    for (int k = 0; k < st.nbuf; ++k) mbar_init(&ts->bars[k], 1u);
    fence_mbar_init();
  }
  __syncthreads();
  int64_t g = g0;
  while (g < g1) {
    // the unit holding tile g and this CTA's tiles of it
    int b = 0;
    {
      int lo = 0, hi = sp.B - 1;  // last b with Hkv * prefix[b] <= g
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((int64_t)sp.Hkv * sp.ws.prefix[mid] <= g) lo = mid; else hi = mid - 1;
      }
      b = lo;
    }
    const int nb = sp.ws.prefix[b + 1] - sp.ws.prefix[b];
    const int64_t base = (int64_t)sp.Hkv * sp.ws.prefix[b];
    const int kvh = (int)((g - base) / nb);
    const int64_t ustart = base + (int64_t)kvh * nb;  // the unit's first tile
    const int i0 = (int)(g - ustart);
    const int i1 = (int)(min(g1, ustart + nb) - 1 - ustart);  // last tile of the unit in this CTA
    g = ustart + i1 + 1;
    const int64_t u = (int64_t)b * sp.Hkv + kvh;

    UnitInfo ui = unit_info(sp, b, kvh);
    const int t0 = i0 * sp.tile, t1 = min((i1 + 1) * sp.tile, ui.nC);
    if (!ui.select || t0 >= t1) continue;
    const float *lg = sp.ws.logits + (size_t)u * sp.ustride * G;
    float *sc = sp.ws.scores + (size_t)u * sp.ustride;
    const int nchunks = tail_issue_first<G>(lg, t0, t1, ts, st);  // in flight during the LSE
    mark_records(ui, ts->ok);
    const float *rec0 = sp.ws.records + (size_t)u * sp.R * RS;
    unit_lse<G, D>(rec0, ui, sp.c, ts->lse, ts->M, ts->L, ts->red);
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) ts->hist[i] = 0u;
    __syncthreads();
    if (!tail_score_range<G>(lg, sc, t0, t1, nchunks, sp.c, ts->lse, ts, st)) {
      if (threadIdx.x == 0) set_error(sp.ws.err, kErrGridWait);
      return;  // a copy never landed: its buffer may still be written
    }
    uint32_t *gh = sp.ws.hist + (size_t)u * kHistBins;
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
      if (ts->hist[i]) atomicAdd(gh + i, ts->hist[i]);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      // CTAs of this unit with selectable positions: the last of them to
      // arrive finds the threshold
      int nsel = 0;
      for (int j = 0; j < ui.nseg; ++j) {
        if (!ui.rec_ok(j)) continue;
        const int64_t ft = max(ui.part.start(ui.c0 + j), ui.U) - ui.U;  // its first tile of the unit
        if (ft * sp.tile < ui.nC) ++nsel;
      }
      ts->last = atomicAdd(sp.ws.ticket + u, 1u) == (uint32_t)(nsel - 1);
    }
    __syncthreads();
    if (!ts->last) continue;
    __threadfence();
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) ts->hist[i] = __ldcg(gh + i);
    __syncthreads();
    int above;
    int bin = find_threshold_bin(ts->hist, kHistBins, sp.k_global, &above, ts->warp, ts->res);
    if (bin < kTrustBin) bin = rescale_unit<G>(sp, ui.nC, lg, sc, ts->hist, ts->lse, bin, &above, ts->warp, ts->res);
    if (threadIdx.x == 0) sp.ws.thr[u] = make_int2(bin, above);
    if (threadIdx.x < G) sp.ws.lse[u * kMaxGroup + threadIdx.x] = ts->lse[threadIdx.x];
    __syncthreads();
  }
  // the attention outputs: combine piece (unit, 256 elements) k goes to CTA
  // k mod grid, each with the unit's max and normaliser from its records
  const int64_t npieces = (int64_t)sp.B * sp.Hkv * sp.ncomb;
  for (int64_t k = blockIdx.x; k < npieces; k += gridDim.x) {
    const int64_t u = k / sp.ncomb;
    const int comb = (int)(k % sp.ncomb);
    const int b = (int)(u / sp.Hkv), kvh = (int)(u % sp.Hkv);
    UnitInfo ui = unit_info(sp, b, kvh);
    if (ui.nseg == 0) {  // nothing attended (T = 0): zeros, as the separate call writes them
      const int e0 = comb * kCombineElems, e1 = min(G * D, e0 + kCombineElems);
      for (int e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
        if (sp.out_dtype == 0) static_cast<float *>(sp.out)[u * G * D + e] = 0.f;
        else static_cast<__nv_bfloat16 *>(sp.out)[u * G * D + e] = __float2bfloat16_rn(0.f);
      }
      continue;
    }
    mark_records(ui, ts->ok);
    unit_lse<G, D>(sp.ws.records + (size_t)u * sp.R * RS, ui, sp.c, ts->lse, ts->M, ts->L, ts->red);
    combine_unit<G, D>(sp, ui, u, comb, ts->M, ts->L, ts->hist);
    __syncthreads();
  }
}

// Outputs of the units no CTA attended (sequences with T = 0): zeros, as the
// separate call's combine writes them.  Units are dealt round-robin over CTAs.
__device__ void fused_zero_empty(const ScoreParams &sp) {
  const int64_t units = (int64_t)sp.B * sp.Hkv, n = (int64_t)sp.G * sp.D;
  for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
    const int b = (int)(u / sp.Hkv);
    if (clamp_len(__ldg(sp.seq_lens + b), (int)sp.t_cap) != 0) continue;
    for (int64_t e = threadIdx.x; e < n; e += blockDim.x) {
      if (sp.out_dtype == 0) static_cast<float *>(sp.out)[u * n + e] = 0.f;
      else static_cast<__nv_bfloat16 *>(sp.out)[u * n + e] = __float2bfloat16_rn(0.f);
    }
  }
}

// Group sizes per attention configuration: warps of 8 heads serve groups of
// up to 8, warps of 16 heads groups of 16 and 32 (the host launches the fused
// kernel only for those).
template <int D, int NT>
__device__ void fused_tail_dispatch(const ScoreParams &sp, int64_t g0, int64_t g1, TailSmem *ts, size_t ring_bytes) {
  if constexpr (NT == 1) {
    switch (sp.G) {
      case 1: fused_tail<1, D>(sp, g0, g1, ts, ring_bytes); break;
      case 2: fused_tail<2, D>(sp, g0, g1, ts, ring_bytes); break;
      case 4: fused_tail<4, D>(sp, g0, g1, ts, ring_bytes); break;
      case 8: fused_tail<8, D>(sp, g0, g1, ts, ring_bytes); break;
      default: break;
    }
  } else {
    switch (sp.G) {
      case 16: fused_tail<16, D>(sp, g0, g1, ts, ring_bytes); break;
      case 32: fused_tail<32, D>(sp, g0, g1, ts, ring_bytes); break;
      default: break;
    }
  }
}

}  // namespace

}  // namespace hs2
