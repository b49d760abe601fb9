// hs2_warp_attn.cuh -- one warp's share of an attention tile: 16 K/V rows
// against the G <= 8 query heads of one GQA group, on the tensor cores.
//
// Layout of the contraction (mma.sync m16n8k16, fp32 accumulate):
//   S^T = K Q^T   : A = K (the 16 rows of the slice), B = Q^T (8 heads;
//                   heads >= G zero), so no MMA row is padding.
//   O^T = V^T P^T : A = V^T (16 head dims per m-tile), B = P^T (16 rows x 8
//                   heads).  The S^T accumulator holds rows g, g+8 of heads
//                   2t, 2t+1; one 8x8 register transpose (movmatrix) per half
//                   turns it into the P^T fragment, so P never leaves
//                   registers.
// The tile in shared memory is [panels][rows][128 B] with the 128-byte TMA
// swizzle (16-byte chunk c of row r at chunk c ^ (r & 7)), written either by
// TMA (full layer) or by cp.async (sparse layer).
//
// E4M3 caches: codes are widened to f16 in registers (exact); the query is
// f16 with a per-head power-of-two prescale (exact for its bf16 values); the
// K scale multiplies the logit and the V scale multiplies p, normalised by a
// running maximum so that p stays inside f16's normal range.  The head-dim
// order inside the MMAs is permuted consistently on both operands so every
// shared-memory read is one conflict-free 16-byte load per row.
#pragma once

#include "hs2_common.cuh"

namespace hs2 {

// NSL: 16-row slices per step.  Two slices give the warp two independent
// instruction streams (MMA chains, conversions, exponentials) to interleave.
// NT: 8-head N-tiles per step.  With two (16 heads per warp, MQA-style
// groups), every K and V fragment read from shared memory (and, for E4M3,
// widened) feeds two MMAs instead of being read again by another warp.
template <int D, bool FP8, int NSL = 1, int NT = 1>
struct WarpAttn {
  static_assert(D == 64 || D == 128, "head_dim");
  static_assert(NSL == 1 || NSL == 2, "slices per step");
  static_assert(NT == 1 || NT == 2, "8-head N-tiles per step");
  static_assert(!FP8 || D == 128, "E4M3 path is built for head_dim 128");
  static constexpr int KS = D / 16;  // k-steps of Q K^T and m-tiles of V^T P^T

  uint32_t qa[NT][KS][2];  // B-fragments of Q^T (N-tile n: head 8n + g; zero for heads >= G)
  float qscale[NT][2];     // E4M3: 2^-e undoing the prescale of heads 8n + 2t, 8n + 2t + 1
  float m[NT][2];          // running max of raw logits of heads 8n + 2t, 8n + 2t + 1 (uniform over g)
  float l[NT][2];          // this lane's share of sum exp(c (s - m)) for those heads
  float sig;               // E4M3: running max of the V scale (warp uniform)
  float inv_sig;           // E4M3: 1 / sig (0 while sig is 0)
  float o[NT][KS][4];      // O^T accumulators: dims x heads (8n + 2t, 8n + 2t + 1)

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      m[n][0] = m[n][1] = -INFINITY;
      l[n][0] = l[n][1] = 0.f;
#pragma unroll
      for (int i = 0; i < KS; ++i) o[n][i][0] = o[n][i][1] = o[n][i][2] = o[n][i][3] = 0.f;
    }
    sig = 0.f;
    inv_sig = 0.f;
  }

  // Query of the warp's heads (G <= 8 NT consecutive heads, bf16 [G][D]) into B-fragments.
  __device__ __forceinline__ void load_q(const __nv_bfloat16 *q, int G) {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const uint32_t *q32 = reinterpret_cast<const uint32_t *>(q);
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int hh = 8 * n + g;  // this lane's head of N-tile n
      if constexpr (!FP8) {
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          qa[n][kk][0] = hh < G ? __ldg(q32 + ((hh * D + 16 * kk + 2 * t) >> 1)) : 0u;
          qa[n][kk][1] = hh < G ? __ldg(q32 + ((hh * D + 16 * kk + 8 + 2 * t) >> 1)) : 0u;
        }
        qscale[n][0] = qscale[n][1] = 1.f;
      } else {
        // k-step kk of lane t covers dims 32t + 4kk + {0,1} (MMA k = 2t, 2t+1)
        // and 32t + 4kk + {2,3} (MMA k = 2t+8, 2t+9).
        float v[KS][4];
        float amax = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          uint2 w = hh < G ? __ldg(reinterpret_cast<const uint2 *>(q + hh * D + 32 * t + 4 * kk)) : make_uint2(0, 0);
          v[kk][0] = __uint_as_float(w.x << 16);
          v[kk][1] = __uint_as_float(w.x & 0xFFFF0000u);
          v[kk][2] = __uint_as_float(w.y << 16);
          v[kk][3] = __uint_as_float(w.y & 0xFFFF0000u);
#pragma unroll
          for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(v[kk][e]));
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const int e = amax > 0.f ? 14 - ilogbf(amax) : 0;
        const float up = ldexpf(1.f, e);
        // the logits of this lane belong to heads 8n + 2t, 8n + 2t + 1 (lanes 8t, 8t + 4 hold their exponents)
        qscale[n][0] = ldexpf(1.f, -__shfl_sync(0xffffffffu, e, 8 * t));
        qscale[n][1] = ldexpf(1.f, -__shfl_sync(0xffffffffu, e, 8 * t + 4));
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          qa[n][kk][0] = pack_f16(v[kk][0] * up, v[kk][1] * up);
          qa[n][kk][1] = pack_f16(v[kk][2] * up, v[kk][3] * up);
        }
      }
    }
  }

  // NSL 16-row slices.  kp / vp: shared addresses of panel 0 of the K / V
  // tile; pstride: bytes between panels; row0: first row of the first slice
  // inside the panel (slice sl starts at row0 + 16 sl); vmask: bit r set when
  // row row0 + r holds a real position; c: 1/sqrt(D) in the logit domain.
  // logit_dst (or nullptr): raw logits of these rows for the G heads of this
  // warp, row r at logit_dst + r * ldl.  ks / vs (E4M3): the rows' K / V
  // scales in shared memory.
  __device__ __forceinline__ void step(uint32_t kp, uint32_t vp, uint32_t pstride, int row0, uint32_t vmask,
                                       float c, float *logit_dst, int G, const float *ks, const float *vs,
                                       int ldl = -1) {
    if (ldl < 0) ldl = G;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    // two accumulator chains per slice and N-tile (even / odd k-steps) halve
    // the dependent-MMA latency; their fp32 sum is the logit
    float s[NSL][NT][4], s2[NSL][NT][4];
#pragma unroll
    for (int sl = 0; sl < NSL; ++sl)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[sl][n][e] = s2[sl][n][e] = 0.f;

    // ---- S^T = K Q^T
    if constexpr (!FP8) {
      // matrices of one ldmatrix.x4: rows 0-7 / 8-15 x dims 0-7, then 8-15
      const int row = row0 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        const int cb = (16 * kk + 8 * (lane >> 4)) * 2;  // byte column
#pragma unroll
        for (int sl = 0; sl < NSL; ++sl) {
          uint32_t r[4];
          ldsm_x4(r, swz(kp + (cb >> 7) * pstride, row + 16 * sl, (cb & 127) >> 4));
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            if (kk & 1) mma_bf16(s2[sl][n], r[0], r[1], r[2], r[3], qa[n][kk][0], qa[n][kk][1]);
            else mma_bf16(s[sl][n], r[0], r[1], r[2], r[3], qa[n][kk][0], qa[n][kk][1]);
          }
        }
      }
    } else {
      uint32_t w[NSL][2][8];
#pragma unroll
      for (int sl = 0; sl < NSL; ++sl)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int row = row0 + 16 * sl + 8 * j + g;
          lds128(*reinterpret_cast<uint32_t(*)[4]>(&w[sl][j][0]), swz(kp, row, 2 * t));
          lds128(*reinterpret_cast<uint32_t(*)[4]>(&w[sl][j][4]), swz(kp, row, 2 * t + 1));
        }
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
        for (int sl = 0; sl < NSL; ++sl) {
          uint32_t lo0, hi0, lo1, hi1;
          e4m3x4_to_f16x2x2(w[sl][0][kk], lo0, hi0);
          e4m3x4_to_f16x2x2(w[sl][1][kk], lo1, hi1);
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            if (kk & 1) mma_f16(s2[sl][n], lo0, lo1, hi0, hi1, qa[n][kk][0], qa[n][kk][1]);
            else mma_f16(s[sl][n], lo0, lo1, hi0, hi1, qa[n][kk][0], qa[n][kk][1]);
          }
        }
      }
    }

    // ---- logits, online softmax: x[sl][n][j][h] = row 16 sl + g + 8j, head 8n + 2t + h
    float x[NSL][NT][2][2];
    bool ok[NSL][2];
    float sv[NSL][2];
#pragma unroll
    for (int sl = 0; sl < NSL; ++sl)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int r = 16 * sl + 8 * j + g;
        ok[sl][j] = ((vmask >> r) & 1u) != 0u;
        sv[sl][j] = 0.f;
        float kj = 1.f;
        if constexpr (FP8) {
          kj = ok[sl][j] ? ks[r] : 0.f;
          sv[sl][j] = ok[sl][j] ? vs[r] : 0.f;
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          x[sl][n][j][0] = s[sl][n][2 * j] + s2[sl][n][2 * j];
          x[sl][n][j][1] = s[sl][n][2 * j + 1] + s2[sl][n][2 * j + 1];
          if constexpr (FP8) {
            x[sl][n][j][0] *= kj * qscale[n][0];
            x[sl][n][j][1] *= kj * qscale[n][1];
          }
        }
      }
    if (logit_dst != nullptr) {
      const uint64_t keep = l2_policy_evict_last();  // read back by the score pass
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        if (8 * n + 2 * t >= G) continue;
#pragma unroll
        for (int sl = 0; sl < NSL; ++sl)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (!ok[sl][j]) continue;
            float *dst = logit_dst + (16 * sl + 8 * j + g) * ldl + 8 * n + 2 * t;
            if ((G & 1) == 0) st_global_hint(dst, x[sl][n][j][0], x[sl][n][j][1], keep);
            else {
              st_global_hint(dst, x[sl][n][j][0], keep);
              if (8 * n + 2 * t + 1 < G) st_global_hint(dst + 1, x[sl][n][j][1], keep);
            }
          }
      }
    }
    // Lazy rescaling: the reference m only moves when a logit would lift
    // exp(c (x - m)) above 2^8 (and sig when a V scale exceeds it); p <= 2^8
    // is exact in the MMA's P operand, and (m, l, o) stay consistent, so the
    // result equals an eager online softmax.  The common case costs one vote.
    const float cl = c * 1.44269504088896341f;  // exp(c x) = 2^(x cl)
    const float thr = 8.f / cl;
    float mloc[NT][2], sloc = 0.f;
    bool grow = false;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      mloc[n][0] = mloc[n][1] = -INFINITY;
#pragma unroll
      for (int sl = 0; sl < NSL; ++sl)
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int h = 0; h < 2; ++h) mloc[n][h] = fmaxf(mloc[n][h], ok[sl][j] ? x[sl][n][j][h] : -INFINITY);
      grow = grow || mloc[n][0] > m[n][0] + thr || mloc[n][1] > m[n][1] + thr;
    }
#pragma unroll
    for (int sl = 0; sl < NSL; ++sl)
#pragma unroll
      for (int j = 0; j < 2; ++j) sloc = fmaxf(sloc, sv[sl][j]);
    grow = grow || (FP8 && sloc > sig);
    float alpha[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n) alpha[n][0] = alpha[n][1] = 1.f;
    if (__any_sync(0xffffffffu, grow)) {
      float beta = 1.f;
      if constexpr (FP8) {
        float smax = fmaxf(sloc, __shfl_xor_sync(0xffffffffu, sloc, 4));
        smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 8));
        smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, 16));
        const float sig_new = fmaxf(sig, smax);
        if (sig_new > sig) {
          inv_sig = __frcp_rn(sig_new);
          beta = sig * inv_sig;
          sig = sig_new;
        }
      }
      float f[NT][2];
      bool any_f = false;
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // max over the rows: lanes of equal t
          float mx = fmaxf(mloc[n][h], __shfl_xor_sync(0xffffffffu, mloc[n][h], 4));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
          const float m_new = fmaxf(m[n][h], mx);
          if (m_new != m[n][h]) alpha[n][h] = ex2_approx((m[n][h] - m_new) * cl);  // 0 when m was -inf
          m[n][h] = m_new;
          f[n][h] = alpha[n][h] * beta;
          any_f = any_f || f[n][h] != 1.f;
        }
      // rescale the O^T columns of heads 8n + 2t, 8n + 2t + 1
      if (__any_sync(0xffffffffu, any_f)) {
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
          for (int i = 0; i < KS; ++i) {
            o[n][i][0] *= f[n][0];
            o[n][i][1] *= f[n][1];
            o[n][i][2] *= f[n][0];
            o[n][i][3] *= f[n][1];
          }
      }
    }
    uint32_t pb[NSL][NT][2];  // P^T fragments: the transposed 8x8 halves (rows 0-7, 8-15 x heads)
    float lsum[NT][2];
#pragma unroll
    for (int n = 0; n < NT; ++n) lsum[n][0] = lsum[n][1] = 0.f;
#pragma unroll
    for (int sl = 0; sl < NSL; ++sl)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          float pr[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {  // the difference first: dominant terms exact
            pr[h] = ok[sl][j] ? ex2_approx((x[sl][n][j][h] - m[n][h]) * cl) : 0.f;
            lsum[n][h] += pr[h];
          }
          if constexpr (FP8) {
            const float w8 = sv[sl][j] * inv_sig;
            pb[sl][n][j] = movmatrix_t(pack_f16(pr[0] * w8, pr[1] * w8));
          } else {
            pb[sl][n][j] = movmatrix_t(pack_bf16(pr[0], pr[1]));
          }
        }
      }
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int h = 0; h < 2; ++h) l[n][h] = l[n][h] * alpha[n][h] + lsum[n][h];

    // ---- O^T += V^T P^T (A rows 2t, 2t+1, 8+2t, 9+2t of each slice)
    const bool full = vmask == (NSL == 2 ? 0xFFFFFFFFu : 0xFFFFu);
    if constexpr (!FP8) {
      uint32_t m01[NSL], m23[NSL];
#pragma unroll
      for (int sl = 0; sl < NSL; ++sl) {
        const uint32_t v0 = (vmask >> (16 * sl + 2 * t)) & 3u, v1 = (vmask >> (16 * sl + 2 * t + 8)) & 3u;
        m01[sl] = ((v0 & 1u) ? 0x0000FFFFu : 0u) | ((v0 & 2u) ? 0xFFFF0000u : 0u);
        m23[sl] = ((v1 & 1u) ? 0x0000FFFFu : 0u) | ((v1 & 2u) ? 0xFFFF0000u : 0u);
      }
      const int row = row0 + (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        const int cb = (16 * mt + ((lane >> 3) & 1) * 8) * 2;
#pragma unroll
        for (int sl = 0; sl < NSL; ++sl) {
          uint32_t a[4];
          ldsm_x4_t(a, swz(vp + (cb >> 7) * pstride, row + 16 * sl, (cb & 127) >> 4));
          if (!full) {  // rows past the end may hold anything, NaN included
            a[0] &= m01[sl];
            a[1] &= m01[sl];
            a[2] &= m23[sl];
            a[3] &= m23[sl];
          }
#pragma unroll
          for (int n = 0; n < NT; ++n) mma_bf16(o[n][mt], a[0], a[1], a[2], a[3], pb[sl][n][0], pb[sl][n][1]);
        }
      }
    } else {
      uint32_t vw[NSL][4][4];  // rows 2t, 2t+1, 2t+8, 2t+9 of each slice: chunk g
      uint32_t b01[NSL], b23[NSL];
#pragma unroll
      for (int sl = 0; sl < NSL; ++sl) {
        const int rb = row0 + 16 * sl + 2 * t;
        lds128(vw[sl][0], swz(vp, rb, g));
        lds128(vw[sl][1], swz(vp, rb + 1, g));
        lds128(vw[sl][2], swz(vp, rb + 8, g));
        lds128(vw[sl][3], swz(vp, rb + 9, g));
        // byte masks: bytes 0,2 come from the even row, bytes 1,3 from the odd row
        const uint32_t v0 = (vmask >> (16 * sl + 2 * t)) & 3u, v1 = (vmask >> (16 * sl + 2 * t + 8)) & 3u;
        b01[sl] = ((v0 & 1u) ? 0x00FF00FFu : 0u) | ((v0 & 2u) ? 0xFF00FF00u : 0u);
        b23[sl] = ((v1 & 1u) ? 0x00FF00FFu : 0u) | ((v1 & 2u) ? 0xFF00FF00u : 0u);
      }
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
#pragma unroll
        for (int sl = 0; sl < NSL; ++sl) {
          uint32_t x01 = prmt(vw[sl][0][mt >> 1], vw[sl][1][mt >> 1], sel);
          uint32_t x23 = prmt(vw[sl][2][mt >> 1], vw[sl][3][mt >> 1], sel);
          if (!full) {
            x01 &= b01[sl];
            x23 &= b23[sl];
          }
          uint32_t a0, a1, a2, a3;
          e4m3x4_to_f16x2x2(x01, a0, a1);
          e4m3x4_to_f16x2x2(x23, a2, a3);
#pragma unroll
          for (int n = 0; n < NT; ++n) mma_f16(o[n][mt], a0, a1, a2, a3, pb[sl][n][0], pb[sl][n][1]);
        }
      }
    }
  }

  // Writes this warp's state to shared scratch: m[8 NT], l[8 NT], o[8 NT][D]
  // (true scale, not yet normalised) at sm, sl, so.  Heads >= G are written
  // too and ignored.
  __device__ __forceinline__ void store(float *sm, float *sl, float *so) const {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // sum over the rows: lanes of equal t
        float lt = l[n][h];
        lt += __shfl_xor_sync(0xffffffffu, lt, 4);
        lt += __shfl_xor_sync(0xffffffffu, lt, 8);
        lt += __shfl_xor_sync(0xffffffffu, lt, 16);
        if (g == 0) {
          sm[8 * n + 2 * t + h] = m[n][h];
          sl[8 * n + 2 * t + h] = lt;
        }
      }
    const float os = FP8 ? sig : 1.f;
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        const int d0 = FP8 ? 16 * g + 2 * mt : 16 * mt + g;
        const int d1 = FP8 ? d0 + 1 : d0 + 8;
        float *on = so + 8 * n * D;
        on[(2 * t) * D + d0] = o[n][mt][0] * os;
        on[(2 * t + 1) * D + d0] = o[n][mt][1] * os;
        on[(2 * t) * D + d1] = o[n][mt][2] * os;
        on[(2 * t + 1) * D + d1] = o[n][mt][3] * os;
      }
  }

  // ---- Merging the states of warps that served the same heads, in registers
  // (a tree over shared memory, one partner at a time).  The saved state is
  // o lane-major (element i of lane L at dst[32 i + L]) followed by (m, l) of
  // the 8 NT heads, which are uniform over g after finish().
  static constexpr int kSaveFloats = NT * 4 * KS + NT * 16 / 32 + 1;  // per lane, rounded up
  static constexpr int kSaveBytes = (NT * 4 * KS * 32 + NT * 16) * 4;

  // Sums l over the rows (lanes of equal t), so every lane holds its heads'
  // whole-warp normaliser, and brings o to its true scale (E4M3: sig = 1
  // afterwards).  Call once before save / absorb / write_record.
  __device__ __forceinline__ void finish() {
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float lt = l[n][h];
        lt += __shfl_xor_sync(0xffffffffu, lt, 4);
        lt += __shfl_xor_sync(0xffffffffu, lt, 8);
        lt += __shfl_xor_sync(0xffffffffu, lt, 16);
        l[n][h] = lt;
      }
    if constexpr (FP8) {
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < KS; ++i)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[n][i][e] *= sig;
      sig = 1.f;
      inv_sig = 1.f;
    }
  }

  __device__ __forceinline__ void save(float *dst) const {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    float *ml = dst + NT * 4 * KS * 32;  // m then l of head 8n + 2t + h at [16 n + 4 h + t], [.. + 8]
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      if (g == 0)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          ml[16 * n + 4 * h + t] = m[n][h];
          ml[16 * n + 8 + 4 * h + t] = l[n][h];
        }
#pragma unroll
      for (int k = 0; k < KS; ++k)
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[32 * (4 * (KS * n + k) + e) + lane] = o[n][k][e];
    }
  }

  // Folds a partner's saved state (same heads, same lane layout) into this one.
  __device__ __forceinline__ void absorb(const float *src, float c) {
    const int lane = threadIdx.x & 31, t = lane & 3;
    const float cl = c * 1.44269504088896341f;
    const float *ml = src + NT * 4 * KS * 32;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float fa[2], fb[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float mb = ml[16 * n + 4 * h + t];
        const float lb = ml[16 * n + 8 + 4 * h + t];
        const float M = fmaxf(m[n][h], mb);
        fa[h] = m[n][h] == -INFINITY ? 0.f : ex2_approx((m[n][h] - M) * cl);
        fb[h] = mb == -INFINITY ? 0.f : ex2_approx((mb - M) * cl);
        l[n][h] = l[n][h] * fa[h] + lb * fb[h];
        m[n][h] = M;
      }
#pragma unroll
      for (int k = 0; k < KS; ++k)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          o[n][k][e] = o[n][k][e] * fa[e & 1] + src[32 * (4 * (KS * n + k) + e) + lane] * fb[e & 1];
    }
  }

  // Writes the (finished) state of heads [0, G) into a record of Gtot heads
  // m[Gtot], l[Gtot], o[Gtot][D] at rec (global), as heads hoff + h.
  __device__ __forceinline__ void write_record(float *rec, int G, int hoff, int Gtot) const {
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int hh = 8 * n + 2 * t + h;
        if (g == 0 && hh < G) {
          rec[hoff + hh] = m[n][h];
          rec[Gtot + hoff + hh] = l[n][h];
        }
      }
    float *ro = rec + 2 * Gtot + hoff * D;
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        const int d0 = FP8 ? 16 * g + 2 * mt : 16 * mt + g;
        const int d1 = FP8 ? d0 + 1 : d0 + 8;
        const int h0 = 8 * n + 2 * t;
        if (h0 < G) {
          ro[h0 * D + d0] = o[n][mt][0];
          ro[h0 * D + d1] = o[n][mt][2];
        }
        if (h0 + 1 < G) {
          ro[(h0 + 1) * D + d0] = o[n][mt][1];
          ro[(h0 + 1) * D + d1] = o[n][mt][3];
        }
      }
  }
};

// Merges NW warp states in shared scratch (stride `wstride` floats per warp:
// m[8], l[8], o[8][D]) of G <= 8 heads into heads hoff .. hoff + G - 1 of a
// record of Gtot heads, m[Gtot], l[Gtot], o[Gtot][D], at `rec` (global or
// shared; Gtot = G, hoff = 0 by default).  Threads tid .. nthreads cooperate.
template <int D>
__device__ __forceinline__ void merge_warp_states(const float *scr, int wstride, int NW, int G, float c,
                                                  float *rec, int tid, int nthreads, int hoff = 0, int Gtot = -1) {
  if (Gtot < 0) Gtot = G;
  for (int h = tid; h < G; h += nthreads) {
    float M = -INFINITY;
    for (int w = 0; w < NW; ++w) M = fmaxf(M, scr[w * wstride + h]);
    float L = 0.f;
    for (int w = 0; w < NW; ++w) {
      const float mw = scr[w * wstride + h];
      if (mw != -INFINITY) L += expf(c * (mw - M)) * scr[w * wstride + 8 + h];
    }
    rec[hoff + h] = M;
    rec[Gtot + hoff + h] = L;
  }
  rec += 2 * Gtot + hoff * D;  // o of head hoff
  // thread -> (dim, first head); each head's warp weights computed once per thread
  const int dim = tid % D, h0 = tid / D, hstep = nthreads / D;
  if (hstep == 0) {  // fewer threads than head dims
    for (int e = tid; e < G * D; e += nthreads) {
      const int h = e / D;
      float M = -INFINITY;
      for (int w = 0; w < NW; ++w) M = fmaxf(M, scr[w * wstride + h]);
      float acc = 0.f;
      for (int w = 0; w < NW; ++w) {
        const float mw = scr[w * wstride + h];
        if (mw != -INFINITY) acc += expf(c * (mw - M)) * scr[w * wstride + 16 + e];
      }
      rec[e] = acc;
    }
    return;
  }
  if (h0 >= hstep * ((G + hstep - 1) / hstep)) return;
  for (int h = h0; h < G; h += hstep) {
    float M = -INFINITY;
    for (int w = 0; w < NW; ++w) M = fmaxf(M, scr[w * wstride + h]);
    float acc = 0.f;
    for (int w = 0; w < NW; ++w) {
      const float mw = scr[w * wstride + h];
      if (mw != -INFINITY) acc += expf(c * (mw - M)) * scr[w * wstride + 16 + h * D + dim];
    }
    rec[h * D + dim] = acc;
  }
}

}  // namespace hs2
