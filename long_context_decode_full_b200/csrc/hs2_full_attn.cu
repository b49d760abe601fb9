// hs2_full_attn.cu -- the full-attention layer of a Hybrid Block, split over
// the context (HySparse2 announcement, "KV Reuse" section: the full layer
// attends over the whole shared KV cache and its attention scores drive the
// token selection).
//
// One persistent CTA per SM walks a balanced share of the (sequence, kv head,
// tile) space.  A producer warp streams K and V tiles with TMA bulk-tensor
// loads into a ring of shared-memory stages (mbarrier full/empty pairs, every
// wait bounded); for E4M3 caches a second producer warp gathers the per-token
// scales with cp.async at the same time.  Consumer warps each take one or two
// 16-row slices of a tile, run K Q^T and V^T P^T on the tensor cores with an
// online softmax, and store the raw logits (evict-last in L2) that the score
// pass turns into group probabilities.  At the end of
// each segment (a run of tiles of one unit inside one CTA) the consumer warps
// merge their states into one (m, l, o) record.
//
// The fp32 cache variant runs the same partition on the CUDA cores (FFMA), so
// fp32 logits keep full fp32 accuracy.
#include "hs2_fused_tail.cuh"
#include "hs2_internal.h"
#include "hs2_tc.cuh"
#include "hs2_warp_attn.cuh"

namespace hs2 {

namespace {

struct StageMeta {
  int32_t b, kvh, tile, flags;
  int32_t rec, T, pad0, pad1;
};
constexpr int kFirst = 1, kLast = 2, kDone = 4;

// Shared-memory region of the tcgen05 path (after the stage metadata): the
// query as the Q K^T product's B operand (heads x d, 128-byte swizzle), two
// P^T buffers (rows x heads, core matrices of 8 rows x 8 heads), reduction
// scratch, the query's per-head scales (E4M3), the mbarriers and the
// tensor-memory base address; for E4M3 caches then the f16 copies of the
// K tile (two buffers) and of the V tile, in the bf16 tile's layout.
template <bool FP8>
struct TcShared {
  static constexpr int kQ = 0, kP = 8192, kPBuf = 8192, kRed = kP + 2 * kPBuf, kSig = kRed + 4 * 32 * 4;
  static constexpr int kQs = kSig + 16, kBar = kQs + 32 * 4, kEnd = kBar + 12 * 8;
  static constexpr int kK16 = (kEnd + 1023) / 1024 * 1024, kV16 = kK16 + 2 * 32768;
  static constexpr int kBytes = FP8 ? kV16 + 32768 : kEnd;
  uint8_t *base;
  __device__ uint64_t *s_full() const { return reinterpret_cast<uint64_t *>(base + kBar); }      // [2]
  __device__ uint64_t *p_full() const { return reinterpret_cast<uint64_t *>(base + kBar) + 2; }  // [2]
  __device__ uint64_t *o_done() const { return reinterpret_cast<uint64_t *>(base + kBar) + 4; }  // [2]
  __device__ uint64_t *o_free() const { return reinterpret_cast<uint64_t *>(base + kBar) + 6; }
  __device__ uint64_t *k_full() const { return reinterpret_cast<uint64_t *>(base + kBar) + 7; }  // [2] (E4M3)
  __device__ uint64_t *q_ready() const { return reinterpret_cast<uint64_t *>(base + kBar) + 9; }  // (E4M3)
  __device__ uint32_t *tmem() const { return reinterpret_cast<uint32_t *>(base + kBar + 80); }
  __device__ float *red() const { return reinterpret_cast<float *>(base + kRed); }  // [4 warps][32 heads]
  __device__ float *sig_red() const { return reinterpret_cast<float *>(base + kSig); }  // [4 warps]
  __device__ float *qscale() const { return reinterpret_cast<float *>(base + kQs); }   // [32 heads]
};

template <int D, bool FP8, int NCW, int NSTAGE, int NSL, int NT, bool TC = false>
struct Cfg {
  static constexpr int RPW = 16 * NSL;  // rows per consumer warp
  static constexpr int TILE = RPW * NCW;
  static constexpr int ES = FP8 ? 1 : 2;
  static constexpr int ROWB = D * ES;
  static constexpr int NPANEL = ROWB / 128;
  static constexpr int PANEL = TILE * 128;
  static constexpr int KVB = TILE * ROWB;
  static constexpr int SCB = FP8 ? 2 * TILE * 4 : 0;                // K and V scales of a tile
  static constexpr int STAGE = (2 * KVB + SCB + 1023) / 1024 * 1024;  // K, V, scales; 1 KB aligned for TMA
  static constexpr int WSTRIDE = 16 + 8 * D;
  // NT = 2: one saved warp state per sender of the first merge round
  static constexpr int SLOT = WarpAttn<D, FP8, NSL, NT>::kSaveBytes / 4;
  static constexpr size_t OFF_BAR = (size_t)NSTAGE * STAGE;
  static constexpr size_t OFF_META = OFF_BAR + (2 * NSTAGE + 1) * 8;
  static constexpr size_t OFF_TC = (OFF_META + NSTAGE * sizeof(StageMeta) + 1023) / 1024 * 1024;
  static constexpr size_t OFF_PREFIX = TC ? OFF_TC + TcShared<FP8>::kBytes : OFF_META + NSTAGE * sizeof(StageMeta);
  static size_t bytes(int B) { return OFF_PREFIX + (size_t)(B + 1) * 4 + 1024; }
  static_assert(ROWB % 128 == 0, "rows are whole 128-byte panels");
  // the warps merge a segment's states inside the stage they last read
  static_assert(NT == 2 || (size_t)NCW * WSTRIDE * 4 <= (size_t)STAGE, "merge scratch must fit in one stage");
  static_assert(NT == 1 || (size_t)(NCW / 2) * SLOT * 4 <= (size_t)STAGE, "merge scratch must fit in one stage");
};

__device__ __forceinline__ int64_t slot_of(const int32_t *pt, int max_pages, int ps, int b, int64_t pos) {
  if (pt == nullptr) return (int64_t)b * ps + pos;
  return (int64_t)__ldg(pt + (int64_t)b * max_pages + pos / ps) * ps + pos % ps;
}

// Rendezvous of the consumer warps (bounded, unlike a named barrier, so a
// warp that gave up on a wait cannot leave the others blocked forever).
__device__ __forceinline__ bool consumer_sync(uint64_t *bar, uint32_t &phase) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
  const bool ok = mbar_wait(bar, phase);
  phase ^= 1u;
  return ok;
}

// Tile prefix per sequence: prefix[b] = sum_{b' < b} ceil(T_b' / tile).
__device__ void compute_prefix(const FullParams &p, int32_t *prefix, int tile) {
  const int lane = threadIdx.x & 31;
  int carry = 0;
  for (int base = 0; base < p.B; base += 32) {
    const int b = base + lane;
    int n = 0;
    if (b < p.B) {
      const int T = clamp_len(__ldg(p.seq_lens + b), (int)p.t_cap);
      n = (T + tile - 1) / tile;
    }
    int x = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (b < p.B) prefix[b + 1] = carry + x;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) prefix[0] = 0;
}

// Zero the histogram / ticket / candidate counters of the selection pass.
__device__ __forceinline__ void zero_counters(const FullParams &p, int tid, int nthreads) {
  const int64_t U = (int64_t)p.B * p.Hkv;
  const int64_t words = U * (kHistBins + 2);
  for (int64_t i = (int64_t)blockIdx.x * nthreads + tid; i < words; i += (int64_t)gridDim.x * nthreads)
    p.ws.hist[i] = 0u;
}

// Locate the sequence that owns linear tile x (prefix in shared memory).
__device__ __forceinline__ int find_seq(const int32_t *prefix, int B, int Hkv, int64_t x) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {  // last b with Hkv * prefix[b] <= x
    const int mid = (lo + hi + 1) >> 1;
    if ((int64_t)Hkv * prefix[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// producer warps: TMA (+ stage metadata), and for E4M3 the scale gathers
template <bool FP8>
constexpr int kProducerWarps = FP8 ? 2 : 1;


// ------------------------------------------------------------ tcgen05 path
// Groups of 16 or 32 query heads over a bf16 cache with d 128 (MQA-style):
// the group is a real M x N tile, so both products of a 128-row tile run on
// tcgen05 with the accumulators in tensor memory.  One warp issues the MMAs
// (one elected lane): S^T = K Q^T (M = 128 rows, N = G heads, K = d; A the
// K tile as TMA left it, K-major with the 128-byte swizzle; B the query in
// shared memory, same layout) into one of two S^T buffers, then
// O^T += V^T P^T (M = d, N = G, K = 128 rows; A the V tile read MN-major,
// B the P^T buffer the softmax warps wrote) into O^T.  Four softmax warps
// own one tensor-memory lane (one row of S^T, one dim of O^T) per thread:
// they load the row's G logits, store them for the score pass, keep the
// online softmax (lazy rescaling as in the warp path, decided for the whole
// CTA by a barrier reduction), write p as bf16, and at a segment end read
// O^T and reduce l into the record.  Each loop runs the CTA's tile count, so
// the warps stay in step even when a bounded wait gives up.
constexpr uint32_t kTmemCols = 128;  // S^T buffers at columns 0 and 32, O^T at 64
constexpr int kTcThreads = 128;      // softmax threads (= tensor-memory lanes = tile rows)

__device__ __forceinline__ bool bar_any(bool x) {  // OR over the 128 softmax threads (named barrier 1)
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "barrier.cta.red.or.pred p, 1, 128, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)x)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bar_softmax() { asm volatile("barrier.cta.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void st_global_v4_hint(float *addr, float a, float b, float c, float d, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(addr), "f"(a), "f"(b), "f"(c),
               "f"(d), "l"(pol)
               : "memory");
}

// E4M3 tile rows into the f16 tile layout (two 128-byte-swizzled panels of
// 64 dims): thread r widens row r of the 128-row code tile at `codes`
// (one 128-byte swizzled row per position) into `dst`.  Exact.
__device__ __forceinline__ void tc_widen_row(const uint8_t *codes, uint8_t *dst, int r) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {  // codes 16 c .. 16 c + 15
    const uint4 w = *reinterpret_cast<const uint4 *>(codes + r * 128 + ((c ^ (r & 7)) << 4));
    uint32_t f[8];
    e4m3x4_to_f16x2x2(w.x, f[0], f[1]);
    e4m3x4_to_f16x2x2(w.y, f[2], f[3]);
    e4m3x4_to_f16x2x2(w.z, f[4], f[5]);
    e4m3x4_to_f16x2x2(w.w, f[6], f[7]);
    uint8_t *panel = dst + (c >> 2) * 16384 + r * 128;
    const int c0 = 2 * (c & 3);
    *reinterpret_cast<uint4 *>(panel + ((c0 ^ (r & 7)) << 4)) = make_uint4(f[0], f[1], f[2], f[3]);
    *reinterpret_cast<uint4 *>(panel + (((c0 + 1) ^ (r & 7)) << 4)) = make_uint4(f[4], f[5], f[6], f[7]);
  }
}

template <int NSTAGE, bool FP8>
__device__ void tc_mma_loop(const FullParams &p, uint8_t *smem, uint64_t *full, uint64_t *empty,
                            const StageMeta *meta, const TcShared<FP8> &ts, int64_t ntiles) {
  using C = Cfg<128, FP8, 4, NSTAGE, 2, 2, true>;
  using TS = TcShared<FP8>;
  const int lane = threadIdx.x & 31, G = p.G;
  const uint32_t tmem = *ts.tmem();
  const uint32_t qs = smem_u32(ts.base + TS::kQ);
  const uint32_t fmt = FP8 ? 0u : 1u;  // f16 (widened codes, prescaled query) or bf16
  const uint32_t id_qk = tc::idesc(128, G, fmt, 0, 0), id_pv = tc::idesc(128, G, fmt, 1, 1);
  bool ok = true;
  int segs = 0;             // segments begun
  bool pv_first = false;    // the tile whose PV is next starts a segment
  int pv_stage = 0;
  for (int64_t it = 0; it <= ntiles; ++it) {
    int stage = 0;
    bool first = false;
    if (it < ntiles) {
      stage = (int)(it % NSTAGE);
      ok = ok && mbar_wait(&full[stage], (uint32_t)(it / NSTAGE) & 1u);
      const StageMeta mt = meta[stage];
      first = (mt.flags & kFirst) != 0;
      if (first) {
        // the last Q K^T with the previous query is done before it is replaced
        if (it > 0) ok = ok && mbar_wait(&ts.s_full()[(it - 1) & 1], (uint32_t)((it - 1) >> 1) & 1u);
        if (lane < G) {  // lane h: query head h, 16 chunks of 16 B into its swizzled row
          const uint4 *q = reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(p.q) +
                                                           ((int64_t)mt.b * p.Hkv * G + (int64_t)mt.kvh * G + lane) * 128);
          uint4 v[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) v[c] = __ldg(q + c);
          if constexpr (FP8) {
            // f16 with a power-of-two prescale (exact for bf16 values), undone on the logit
            float amax = 0.f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[e] << 16)), fabsf(__uint_as_float(w[e] & 0xFFFF0000u))));
            }
            const int ex = amax > 0.f ? 14 - ilogbf(amax) : 0;
            const float up = ldexpf(1.f, ex);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                w[e] = pack_f16(__uint_as_float(w[e] << 16) * up, __uint_as_float(w[e] & 0xFFFF0000u) * up);
              v[c] = make_uint4(w[0], w[1], w[2], w[3]);
            }
            ts.qscale()[lane] = ldexpf(1.f, -ex);
          }
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int panel = c >> 3, cc = c & 7;
            *reinterpret_cast<uint4 *>(ts.base + TS::kQ + panel * G * 128 + lane * 128 + ((cc ^ (lane & 7)) << 4)) = v[c];
          }
        }
        tc::fence_async_smem();
        __syncwarp();
        if (FP8 && lane == 0) mbar_arrive(ts.q_ready());  // the query's scales, for the softmax warps
      }
      if constexpr (FP8)  // the widened K tile
        ok = ok && mbar_wait(&ts.k_full()[it & 1], (uint32_t)(it >> 1) & 1u);
      tc::fence_after();
      if (lane == 0) {  // S^T = K Q^T into buffer it & 1
        const uint32_t kb = FP8 ? smem_u32(ts.base + TS::kK16) + (uint32_t)(it & 1) * 32768u
                                : smem_u32(smem) + (uint32_t)stage * C::STAGE;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (uint32_t)(kk & 3) * 32;
          const uint64_t a = tc::sdesc(kb + (uint32_t)(kk >> 2) * 16384u + off, 16, 1024, 2);
          const uint64_t b = tc::sdesc(qs + (uint32_t)(kk >> 2) * (uint32_t)(G * 128) + off, 16, 1024, 2);
          tc::mma_f16(tmem + 32u * (uint32_t)(it & 1), a, b, id_qk, kk > 0);
        }
        tc::commit(&ts.s_full()[it & 1]);
      }
      __syncwarp();
    }
    if (it >= 1) {  // O^T += V^T P^T of the previous tile
      const int64_t j = it - 1;
      ok = ok && mbar_wait(&ts.p_full()[j & 1], (uint32_t)(j >> 1) & 1u);
      if (pv_first && segs > 1)  // the previous segment's O^T has been read
        ok = ok && mbar_wait(ts.o_free(), (uint32_t)(segs - 2) & 1u);
      tc::fence_after();
      if (lane == 0) {
        const uint32_t vb = FP8 ? smem_u32(ts.base + TS::kV16) : smem_u32(smem) + (uint32_t)pv_stage * C::STAGE + C::KVB;
        const uint32_t pb = smem_u32(ts.base + TS::kP) + (uint32_t)(j & 1) * TS::kPBuf;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t a = tc::sdesc(vb + (uint32_t)k * 2048, 16384, 1024, 2);  // V^T: MN-major, swizzled
          const uint64_t b = tc::sdesc(pb + (uint32_t)k * 256, 128, 2048, 0);    // P^T: MN-major, core matrices
          tc::mma_f16(tmem + 64u, a, b, id_pv, !(pv_first && k == 0));
        }
        if constexpr (!FP8) tc::commit(&empty[pv_stage]);  // the K/V stage can be refilled
        tc::commit(&ts.o_done()[j & 1]);
      }
      __syncwarp();
    }
    if (it < ntiles) {
      pv_first = first;
      pv_stage = stage;
      if (first) ++segs;
    }
  }
  // the last commit covers every MMA this warp issued: they are done before
  // the tensor memory is freed (bounded, also after an earlier expiry)
  if (ntiles > 0) mbar_wait(&ts.o_done()[(ntiles - 1) & 1], (uint32_t)((ntiles - 1) >> 1) & 1u, 40000000LL);
  if (!ok && lane == 0) set_error(p.ws.err, kErrFullWait);
}

template <int NSTAGE, bool FP8>
__device__ void tc_softmax_loop(const FullParams &p, uint8_t *smem, uint64_t *full, uint64_t *empty,
                                const StageMeta *meta, const TcShared<FP8> &ts, int64_t ntiles) {
  using C = Cfg<128, FP8, 4, NSTAGE, 2, 2, true>;
  using TS = TcShared<FP8>;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, G = p.G;
  const uint32_t tmem = *ts.tmem();
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;  // warp w reads lanes 32 w .. 32 w + 31
  const float cl = p.c * 1.44269504088896341f;            // exp(c x) = 2^(x cl)
  const float thr = 8.f / cl;                              // p stays <= 2^8
  float m[32], l[32], qsc[32];
  float sig = 0.f, inv_sig = 0.f;                          // E4M3: running max of the V scale
  bool ok = true;
  int segs = 0;
  float *red = ts.red();
#pragma unroll
  for (int h = 0; h < 32; ++h) qsc[h] = 1.f;
  if constexpr (FP8) {  // the first tile's K codes, widened
    if (ntiles > 0) {
      ok = ok && mbar_wait(&full[0], 0u);
      tc_widen_row(smem, ts.base + TS::kK16, tid);
      tc::fence_async_smem();
      mbar_arrive(&ts.k_full()[0]);
    }
  }
  for (int64_t it = 0; it < ntiles; ++it) {
    const int stage = (int)(it % NSTAGE);
    ok = ok && mbar_wait(&full[stage], (uint32_t)(it / NSTAGE) & 1u);
    const StageMeta mt = meta[stage];
    const bool first = (mt.flags & kFirst) != 0, last = (mt.flags & kLast) != 0;
    if (first) {
#pragma unroll
      for (int h = 0; h < 32; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
      }
      sig = 0.f;
      inv_sig = 0.f;
      if constexpr (FP8) {  // the query's per-head scales
        ok = ok && mbar_wait(ts.q_ready(), (uint32_t)segs & 1u);
#pragma unroll
        for (int h = 0; h < 32; ++h) qsc[h] = h < G ? ts.qscale()[h] : 1.f;
      }
      ++segs;
    }
    if constexpr (FP8) {  // the next tile's K codes, widened, while this tile's S^T is computed
      if (it + 1 < ntiles) {
        const int st1 = (int)((it + 1) % NSTAGE);
        ok = ok && mbar_wait(&full[st1], (uint32_t)((it + 1) / NSTAGE) & 1u);
        tc_widen_row(smem + (size_t)st1 * C::STAGE, ts.base + TS::kK16 + (size_t)((it + 1) & 1) * 32768, tid);
        tc::fence_async_smem();
        mbar_arrive(&ts.k_full()[(it + 1) & 1]);
      }
    }
    const int pos = mt.tile * C::TILE + tid;
    const bool valid = pos < mt.T;
    float kr = 1.f, vr = 0.f;  // E4M3: this row's K and V scales
    if constexpr (FP8) {
      const float *sc = reinterpret_cast<const float *>(smem + (size_t)stage * C::STAGE + 2 * C::KVB);
      kr = valid ? sc[tid] : 0.f;
      vr = valid ? sc[C::TILE + tid] : 0.f;
    }
    ok = ok && mbar_wait(&ts.s_full()[it & 1], (uint32_t)(it >> 1) & 1u);
    tc::fence_after();
    float x[32];
    tc::ld32(tmem + lane_base + 32u * (uint32_t)(it & 1), x);
    if constexpr (FP8) {
#pragma unroll
      for (int h = 0; h < 32; ++h) x[h] *= kr * qsc[h];
    }
    const int64_t u = (int64_t)mt.b * p.Hkv + mt.kvh;
    if (valid) {  // raw logits for the score pass (evict-last in L2)
      float *dst = p.ws.logits + (u * p.ustride + pos) * G;
      const uint64_t keep = l2_policy_evict_last();
#pragma unroll
      for (int h4 = 0; h4 < 8; ++h4)
        if (4 * h4 < G) st_global_v4_hint(dst + 4 * h4, x[4 * h4], x[4 * h4 + 1], x[4 * h4 + 2], x[4 * h4 + 3], keep);
    }
    bool grow = FP8 && vr > sig;
#pragma unroll
    for (int h = 0; h < 32; ++h) grow = grow || (h < G && valid && x[h] > m[h] + thr);
    if (bar_any(grow)) {
      // the new per-head maxima (and E4M3: the V scales' maximum) over the tile, for the whole CTA
#pragma unroll
      for (int h = 0; h < 32; ++h) {
        if (h >= G) break;
        const float v = warp_max(valid ? x[h] : -INFINITY);
        if (lane == 0) red[warp * 32 + h] = v;
      }
      if constexpr (FP8) {
        const float v = warp_max(vr);
        if (lane == 0) ts.sig_red()[warp] = v;
      }
      bar_softmax();
      float beta = 1.f;
      if constexpr (FP8) {
        const float smax = fmaxf(fmaxf(ts.sig_red()[0], ts.sig_red()[1]), fmaxf(ts.sig_red()[2], ts.sig_red()[3]));
        if (smax > sig) {
          const float inv_new = __frcp_rn(smax);
          beta = sig * inv_new;
          sig = smax;
          inv_sig = inv_new;
        }
      }
      float f[32];
#pragma unroll
      for (int h = 0; h < 32; ++h) {
        float alpha = 1.f;
        if (h < G) {
          const float mx = fmaxf(fmaxf(red[h], red[32 + h]), fmaxf(red[64 + h], red[96 + h]));
          const float m_new = fmaxf(m[h], mx);
          if (m_new != m[h]) alpha = m[h] == -INFINITY ? 0.f : ex2_approx((m[h] - m_new) * cl);
          m[h] = m_new;
          l[h] *= alpha;
        }
        f[h] = alpha * beta;
      }
      bar_softmax();  // red is read before it is written again
      if (!first) {   // O^T holds this segment's earlier tiles: rescale its columns
        ok = ok && mbar_wait(&ts.o_done()[(it - 1) & 1], (uint32_t)((it - 1) >> 1) & 1u);
        tc::fence_after();
        float o[32];
        tc::ld32(tmem + lane_base + 64u, o);
#pragma unroll
        for (int h = 0; h < 32; ++h) o[h] *= f[h];
        tc::st32(tmem + lane_base + 64u, o);
      }
    }
    // p = 2^((x - m) cl); l sums it; the P^T operand carries p (bf16), or
    // p times the row's V scale over sig (f16, E4M3)
    const float w8 = FP8 ? vr * inv_sig : 1.f;
    uint32_t pk[16];
#pragma unroll
    for (int h2 = 0; h2 < 16; ++h2) {
      float p0 = 0.f, p1 = 0.f;
      if (valid && 2 * h2 < G) {
        p0 = ex2_approx((x[2 * h2] - m[2 * h2]) * cl);
        p1 = ex2_approx((x[2 * h2 + 1] - m[2 * h2 + 1]) * cl);
        l[2 * h2] += p0;
        l[2 * h2 + 1] += p1;
      }
      pk[h2] = FP8 ? pack_f16(p0 * w8, p1 * w8) : pack_bf16(p0, p1);
    }
    if (FP8 ? it >= 1 : it >= 2)  // E4M3: the V copy and P^T buffers' previous tile has been multiplied
      ok = ok && mbar_wait(&ts.o_done()[FP8 ? (it - 1) & 1 : it & 1],
                           (uint32_t)((FP8 ? it - 1 : it - 2) >> 1) & 1u);
    if constexpr (FP8) {  // this tile's V codes, widened (zeros past the end), then the stage is free
      uint8_t *v16 = ts.base + TS::kV16;
      if (valid) {
        tc_widen_row(smem + (size_t)stage * C::STAGE + C::KVB, v16, tid);
      } else {
#pragma unroll
        for (int pn = 0; pn < 2; ++pn)
#pragma unroll
          for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(v16 + pn * 16384 + tid * 128 + c * 16) = make_uint4(0, 0, 0, 0);
      }
    }
    uint8_t *pbuf = ts.base + TS::kP + (size_t)(it & 1) * TS::kPBuf;
#pragma unroll
    for (int n8 = 0; n8 < 4; ++n8)
      if (8 * n8 < G)
        *reinterpret_cast<uint4 *>(pbuf + n8 * 2048 + tid * 16) =
            make_uint4(pk[4 * n8], pk[4 * n8 + 1], pk[4 * n8 + 2], pk[4 * n8 + 3]);
    if constexpr (!FP8) {
      if (!valid) {  // rows past the end may hold anything (NaN included): zero the V row
        uint8_t *vrow = smem + (size_t)stage * C::STAGE + C::KVB + tid * 128;
#pragma unroll
        for (int pn = 0; pn < 2; ++pn)
#pragma unroll
          for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(vrow + pn * C::PANEL + c * 16) = make_uint4(0, 0, 0, 0);
      }
    }
    tc::fence_async_smem();
    tc::fence_before();
    if constexpr (FP8) mbar_arrive(&empty[stage]);  // codes and scales of this tile are consumed
    mbar_arrive(&ts.p_full()[it & 1]);
    if (last) {  // segment end: the record from O^T, m and the rows' l
      ok = ok && mbar_wait(&ts.o_done()[it & 1], (uint32_t)(it >> 1) & 1u);
      tc::fence_after();
      float o[32];
      tc::ld32(tmem + lane_base + 64u, o);
#pragma unroll
      for (int h = 0; h < 32; ++h) {
        if (h >= G) break;
        const float v = warp_sum(l[h]);
        if (lane == 0) red[warp * 32 + h] = v;
      }
      bar_softmax();
      if (mt.rec >= 0) {
        float *rec = p.ws.records + (size_t)mt.rec * G * 130;
        const float os = FP8 ? sig : 1.f;
#pragma unroll
        for (int h = 0; h < 32; ++h)
          if (h < G) rec[2 * G + h * 128 + tid] = o[h] * os;
        if (tid < G) {
          float mh = -INFINITY;
#pragma unroll
          for (int h = 0; h < 32; ++h)
            if (h == tid) mh = m[h];
          rec[tid] = mh;
          rec[G + tid] = (red[tid] + red[32 + tid]) + (red[64 + tid] + red[96 + tid]);
        }
      }
      tc::fence_before();
      bar_softmax();  // red and O^T are read
      mbar_arrive(ts.o_free());
    }
  }
  if (!ok) set_error(p.ws.err, kErrFullWait);
}

// The attention pass of one CTA; with FUSED the CTA then runs the score pass
// of the selection (hs2_fused_tail.cuh) over the tiles it attended.
template <int D, bool FP8, int NCW, int NSTAGE, int NSL, int NT, bool FUSED, bool TC = false>
__device__ __forceinline__ void full_attn_body(const CUtensorMap &tmk, const CUtensorMap &tmv, const FullParams &p,
                                               const ScoreParams *sp) {
  using C = Cfg<D, FP8, NCW, NSTAGE, NSL, NT, TC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  uint64_t *empty = full + NSTAGE;
  uint64_t *cbar = empty + NSTAGE;  // consumer-warp rendezvous at segment ends
  StageMeta *meta = reinterpret_cast<StageMeta *>(smem + C::OFF_META);
  int32_t *prefix = reinterpret_cast<int32_t *>(smem + C::OFF_PREFIX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kMmaWarps = TC ? 1 : 0;  // the tcgen05 path's MMA-issuing warp follows the consumers
  const bool producer = warp >= NCW + kMmaWarps;
  const bool tma_role = warp == NCW + kMmaWarps;  // the other producer warp (E4M3) gathers scales
  const bool mma_role = TC && warp == NCW;
  const TcShared<FP8> ts{smem + C::OFF_TC};

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], FP8 ? 33u : 1u);
      // tcgen05: one commit releases a stage (E4M3: the softmax threads, once its codes are widened)
      mbar_init(&empty[s], TC ? (FP8 ? (uint32_t)kTcThreads : 1u) : (uint32_t)NCW);
    }
    mbar_init(cbar, (uint32_t)NCW);
    if constexpr (TC) {
      for (int k = 0; k < 2; ++k) {
        mbar_init(&ts.s_full()[k], 1u);
        mbar_init(&ts.p_full()[k], (uint32_t)kTcThreads);
        mbar_init(&ts.o_done()[k], 1u);
      }
      mbar_init(ts.o_free(), (uint32_t)kTcThreads);
      for (int k = 0; k < 2; ++k) mbar_init(&ts.k_full()[k], (uint32_t)kTcThreads);
      mbar_init(ts.q_ready(), 1u);
    }
    fence_mbar_init();
  }
  if (tma_role && lane == 0) {
    prefetch_tensormap(&tmk);
    prefetch_tensormap(&tmv);
  }
  griddep_wait();               // inputs and workspace are free from here on
  griddep_launch_dependents();  // the score kernel may be scheduled as SMs free up
  if (tma_role) {
    compute_prefix(p, prefix, C::TILE);
  } else if (warp < NCW) {
    zero_counters(p, threadIdx.x, NCW * 32);
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i <= p.B; i += blockDim.x) p.ws.prefix[i] = prefix[i];

  const int64_t total = (int64_t)p.Hkv * prefix[p.B];
  if (total == 0) {  // every sequence is empty (the same for all CTAs: no barrier)
    if constexpr (FUSED) fused_zero_empty(*sp);
    return;
  }
  const Partition part{total, p.N};
  const int64_t g0 = part.start(blockIdx.x), g1 = part.start(blockIdx.x + 1);
  if constexpr (TC) {  // tensor memory for the S^T buffers and O^T
    if (mma_role) {
      tc::tmem_alloc(ts.tmem(), kTmemCols);
      tc::tmem_relinquish();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
  }

  [&]() {  // producers and consumers; both return here when their work is done
  if (producer) {
    // ------------------------------------------------------------ producers
    // Boxes of RB rows (one page, or the whole tile when pages are larger).
    // Lane L caches the first slot of CTA-local box cache_base + L, so page
    // table reads are issued 32 at a time instead of one per box.  Both
    // producer warps walk the same tiles; the (sequence, kv head, tile)
    // coordinates advance incrementally.
    const int RB = p.page_table ? min(C::TILE, p.page_size) : C::TILE;
    const int BPT = C::TILE / RB;  // boxes per tile (<= 8)
    int64_t cache_base = -(int64_t)64;
    int my_slot = -1;
    int it = 0;
    int b = 0, kvh = 0, i = 0, nb = 1, T = 0;
    if (g0 < g1) {
      b = find_seq(prefix, p.B, p.Hkv, g0);
      nb = prefix[b + 1] - prefix[b];
      const int64_t r = g0 - (int64_t)p.Hkv * prefix[b];
      kvh = (int)(r / nb);
      i = (int)(r % nb);
      T = clamp_len(__ldg(p.seq_lens + b), (int)p.t_cap);
    }
    bool ok = true;
    for (int64_t g = g0; g < g1; ++g, ++it) {
      const int64_t box0 = (g - g0) * BPT;
      if (box0 + BPT > cache_base + 32) {  // refill: lane L -> box box0 + L
        cache_base = box0;
        const int64_t bx = box0 + lane, gl = g0 + bx / BPT;
        my_slot = -1;
        if (gl < g1) {
          const int bl = find_seq(prefix, p.B, p.Hkv, gl);
          const int nbl = prefix[bl + 1] - prefix[bl];
          const int il = (int)((gl - (int64_t)p.Hkv * prefix[bl]) % nbl);
          const int pos = il * C::TILE + (int)(bx % BPT) * RB;
          const int Tl = clamp_len(__ldg(p.seq_lens + bl), (int)p.t_cap);
          if (pos < Tl) {
            const int64_t sl = slot_of(p.page_table, p.max_pages, p.page_size, bl, pos);
            my_slot = (sl >= 0 && sl < p.num_slots) ? (int)sl : -1;
          }
        }
      }
      const int stage = it % NSTAGE;
      if (it >= NSTAGE && !mbar_wait(&empty[stage], ((it / NSTAGE) - 1) & 1)) {
        set_error(p.ws.err, kErrEmptyWait);
        ok = false;
        break;
      }
      const int p0 = i * C::TILE;
      const int cl0 = (int)(box0 - cache_base);  // cache lane of this tile's first box
      if (!tma_role) {
        if constexpr (FP8) {  // per-token scales of the tile's rows
          float *ks = reinterpret_cast<float *>(smem + (size_t)stage * C::STAGE + 2 * C::KVB);
#pragma unroll
          for (int k = 0; k < C::TILE / 32; ++k) {
            const int rr = lane + 32 * k;
            const int bs = __shfl_sync(0xffffffffu, my_slot, cl0 + rr / RB);
            if (p0 + rr < T && bs >= 0) {
              const int64_t slot = (int64_t)bs + rr % RB;
              cp_async_4(smem_u32(ks + rr), p.k_scale + slot * p.Hkv + kvh);
              cp_async_4(smem_u32(ks + C::TILE + rr), p.v_scale + slot * p.Hkv + kvh);
            }
          }
          cp_async_mbar_arrive_noinc(&full[stage]);
        }
      } else {
        int box_slot[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) box_slot[k] = __shfl_sync(0xffffffffu, my_slot, min(cl0 + k, 31));
        if (lane == 0) {
          const int64_t U = (int64_t)p.Hkv * prefix[b] + (int64_t)kvh * nb;  // first tile of the unit
          const int64_t j = blockIdx.x - part.cfirst(U);
          const int64_t u = (int64_t)b * p.Hkv + kvh;
          StageMeta mt;
          mt.b = b;
          mt.kvh = kvh;
          mt.tile = i;
          mt.flags = ((i == 0 || g == g0) ? kFirst : 0) | ((i == nb - 1 || g == g1 - 1) ? kLast : 0);
          mt.rec = (j >= 0 && j < p.R) ? (int)(u * p.R + j) : -1;
          if (mt.rec < 0) set_error(p.ws.err, kErrRecord);
          mt.T = T;
          meta[stage] = mt;
          const int nbox = min(BPT, (T - p0 + RB - 1) / RB);
          mbar_arrive_expect_tx(&full[stage], (uint32_t)nbox * 2u * RB * C::ROWB);
          const uint32_t kdst = sbase + stage * C::STAGE, vdst = kdst + C::KVB;
          const uint64_t once = p.kv_evict_first ? l2_policy_evict_first() : l2_policy_evict_normal();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            if (k >= nbox) break;
            // a slot outside the cache (bad page id) loads from row 2^31 - 1 .. : out of
            // the tensor, so TMA fills zeros and the transfer still completes
            const int slot = box_slot[k] >= 0 ? box_slot[k] : 0x7FFFFFFF - RB;
#pragma unroll
            for (int pn = 0; pn < C::NPANEL; ++pn) {
              tma_load_3d_hint(kdst + pn * C::PANEL + k * RB * 128, &tmk, &full[stage], pn * (128 / C::ES), kvh,
                               slot, once);
              tma_load_3d_hint(vdst + pn * C::PANEL + k * RB * 128, &tmv, &full[stage], pn * (128 / C::ES), kvh,
                               slot, once);
            }
          }
        }
      }
      __syncwarp();
      // next tile: (b, kvh, i) in the order of the linear tile index
      if (++i == nb) {
        i = 0;
        if (++kvh == p.Hkv) {
          kvh = 0;
          if (g + 1 < g1) {
            do ++b; while (prefix[b + 1] == prefix[b]);  // sequences without tiles own none
            nb = prefix[b + 1] - prefix[b];
            T = clamp_len(__ldg(p.seq_lens + b), (int)p.t_cap);
          }
        }
      }
    }
    if (ok) {  // end-of-work sentinel
      const int stage = it % NSTAGE;
      if (it >= NSTAGE && !mbar_wait(&empty[stage], ((it / NSTAGE) - 1) & 1)) {
        set_error(p.ws.err, kErrEmptyWait);
      } else if (tma_role) {
        if (lane == 0) {
          meta[stage].flags = kDone;
          mbar_arrive(&full[stage]);
        }
      } else {
        mbar_arrive(&full[stage]);  // the scale warp's 32 arrivals
      }
    }
    return;
  }

  if constexpr (TC) {
    if (mma_role) tc_mma_loop<NSTAGE, FP8>(p, smem, full, empty, meta, ts, g1 - g0);
    else tc_softmax_loop<NSTAGE, FP8>(p, smem, full, empty, meta, ts, g1 - g0);
    return;
  }

  // -------------------------------------------------------------- consumers
  // A warp serves HPW = 8 NT heads (NT MMA N-tiles).  With more heads than
  // that (MQA-style groups) warp w serves head group hg = w % NHG and, of
  // each tile, the row blocks j = w / NHG + k * (NCW / NHG), k < NHG: every
  // head group sees every row of the tile from the same shared-memory stage.
  constexpr int HPW = 8 * NT;
  const int NHG = (p.G + HPW - 1) / HPW, WPG = NCW / NHG;
  const int hg = warp % NHG, wig = warp / NHG;
  const int Gl = min(HPW, p.G - HPW * hg);  // heads of this warp's group
  WarpAttn<D, FP8, NSL, NT> st;
  st.reset();
  uint32_t cphase = 0;
  for (int it = 0;; ++it) {
    const int stage = it % NSTAGE;
    if (!mbar_wait(&full[stage], (it / NSTAGE) & 1)) {
      set_error(p.ws.err, kErrFullWait);
      break;
    }
    const StageMeta mt = meta[stage];
    if (mt.flags & kDone) break;
    const int64_t u = (int64_t)mt.b * p.Hkv + mt.kvh;
    if (mt.flags & kFirst) {
      st.reset();
      st.load_q(reinterpret_cast<const __nv_bfloat16 *>(p.q) +
                    ((int64_t)mt.b * p.Hkv * p.G + (int64_t)mt.kvh * p.G + HPW * hg) * D,
                Gl);
    }
    const uint32_t kp = sbase + stage * C::STAGE;
    for (int k = 0; k < NHG; ++k) {
      const int j = wig + k * WPG;  // row block of the tile
      const int pos0 = mt.tile * C::TILE + C::RPW * j;
      const int nvalid = max(0, min(C::RPW, mt.T - pos0));
      const uint32_t vmask = nvalid >= 32 ? 0xFFFFFFFFu : ((1u << nvalid) - 1u);
      const float *ks = reinterpret_cast<const float *>(smem + (size_t)stage * C::STAGE + 2 * C::KVB) + C::RPW * j;
      if (nvalid > 0)
        st.step(kp, kp + C::KVB, C::PANEL, C::RPW * j, vmask, p.c,
                p.ws.logits + (u * p.ustride + pos0) * p.G + HPW * hg, Gl, ks, ks + C::TILE, p.G);
    }
    if (mt.flags & kLast) {
      // segment end: merge the warps' states inside this stage, then release it
      if (!consumer_sync(cbar, cphase)) {  // every warp is done reading the tile
        set_error(p.ws.err, kErrFullWait);
        break;
      }
      float *scratch = reinterpret_cast<float *>(smem + (size_t)stage * C::STAGE);
      float *rec = p.ws.records + (size_t)(mt.rec >= 0 ? mt.rec : 0) * p.G * (D + 2);
      if constexpr (NT == 1) {
        float *scr = scratch + warp * C::WSTRIDE;
        st.store(scr, scr + 8, scr + 16);
        if (!consumer_sync(cbar, cphase)) {
          set_error(p.ws.err, kErrFullWait);
          break;
        }
        if (mt.rec >= 0)
          for (int g8 = 0; g8 < NHG; ++g8)  // the warps of head group g8 are g8, g8 + NHG, ...
            merge_warp_states<D>(scratch + g8 * C::WSTRIDE, NHG * C::WSTRIDE, WPG, min(8, p.G - 8 * g8), p.c, rec,
                                 threadIdx.x, NCW * 32, 8 * g8, p.G);
      } else {
        // a tree over the WPG warps of each head group, in registers: in the
        // round of span s, warp wig = 2 s k + s hands its state to 2 s k
        // through slot (hg, k) of the stage; warp wig = 0 writes the record
        st.finish();
        bool sync_ok = true;
        for (int span = 1; span < WPG && sync_ok; span *= 2) {
          const int r = wig % (2 * span);
          float *slot = scratch + (size_t)(hg + NHG * (wig / (2 * span))) * C::SLOT;
          if (r == span) st.save(slot);
          sync_ok = consumer_sync(cbar, cphase);
          if (sync_ok && r == 0 && wig + span < WPG) st.absorb(slot, p.c);
          sync_ok = sync_ok && consumer_sync(cbar, cphase);  // the slots are read before the next round
        }
        if (!sync_ok) {
          set_error(p.ws.err, kErrFullWait);
          break;
        }
        if (wig == 0 && mt.rec >= 0) st.write_record(rec, Gl, HPW * hg, p.G);
      }
      fence_proxy_async_smem();  // before TMA refills the stage
      if (!consumer_sync(cbar, cphase)) {
        set_error(p.ws.err, kErrFullWait);
        break;
      }
      st.reset();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
  }
  }();

  if constexpr (TC) {  // every tcgen05 operation has completed: free the tensor memory
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    if (mma_role) tc::tmem_dealloc(*ts.tmem(), kTmemCols);
  }
  if constexpr (FUSED) {
    // every segment record and logit of the call is written once all CTAs
    // pass the barrier; the K/V stages are idle from here on
    TailSmem *ts = reinterpret_cast<TailSmem *>(smem);
    if (!grid_barrier(p.ws.err + 16, p.ws.err + 32, gridDim.x, &ts->ok_flag)) {
      if (threadIdx.x == 0) set_error(p.ws.err, kErrGridWait);
      return;
    }
    fused_tail_dispatch<D, NT>(*sp, g0, g1, ts, (size_t)C::STAGE * NSTAGE);
  }
}

template <int D, bool FP8, int NCW, int NSTAGE, int NSL, int NT>
__global__ void __launch_bounds__(32 * (NCW + kProducerWarps<FP8>), 1)
    full_attn_mma_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                         const FullParams p) {
  full_attn_body<D, FP8, NCW, NSTAGE, NSL, NT, false>(tmk, tmv, p, nullptr);
}

// Groups of 16 or 32 heads, d 128: the tcgen05 consumers (4 softmax warps,
// 1 MMA warp) and the producers (TMA; E4M3: and the scale gathers).
template <int NSTAGE, bool FP8>
__global__ void __launch_bounds__(32 * (4 + 1 + kProducerWarps<FP8>), 1)
    full_attn_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                        const FullParams p) {
  full_attn_body<128, FP8, 4, NSTAGE, 2, 2, false, true>(tmk, tmv, p, nullptr);
}

template <int NSTAGE>
__global__ void __launch_bounds__(32 * (4 + 1 + 1), 1)
    full_attn_fused_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                              const FullParams p, const ScoreParams sp) {
  full_attn_body<128, false, 4, NSTAGE, 2, 2, true, true>(tmk, tmv, p, &sp);
}

// The fused call: attention, a grid barrier, then the score pass.  Launched
// cooperatively (every CTA resident at once).
template <int D, bool FP8, int NCW, int NSTAGE, int NSL, int NT>
__global__ void __launch_bounds__(32 * (NCW + kProducerWarps<FP8>), 1)
    full_attn_fused_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                           const FullParams p, const ScoreParams sp) {
  full_attn_body<D, FP8, NCW, NSTAGE, NSL, NT, true>(tmk, tmv, p, &sp);
}

// ------------------------------------------------------------ fp32 caches
constexpr int kF32Tile = 64;
constexpr int kF32Warps = 4;

template <int D>
__global__ void __launch_bounds__(32 * kF32Warps) full_attn_f32_kernel(const FullParams p) {
  extern __shared__ float fsm[];
  float *Ks = fsm;                        // [64][D+1]
  float *Vs = Ks + kF32Tile * (D + 1);    // [64][D+1]
  float *Qs = Vs + kF32Tile * (D + 1);    // [8][D]
  int64_t *slots = reinterpret_cast<int64_t *>(Qs + 8 * D);  // the tile's cache slots (-1: none)
  int32_t *prefix = reinterpret_cast<int32_t *>(slots + kF32Tile);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nthr = blockDim.x;
  griddep_wait();
  griddep_launch_dependents();
  if (warp == 0) compute_prefix(p, prefix, kF32Tile);
  zero_counters(p, threadIdx.x, nthr);
  __syncthreads();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i <= p.B; i += nthr) p.ws.prefix[i] = prefix[i];
  const int64_t total = (int64_t)p.Hkv * prefix[p.B];
  if (total == 0) return;
  const Partition part{total, p.N};
  const int64_t g0 = part.start(blockIdx.x), g1 = part.start(blockIdx.x + 1);
  const float *K = static_cast<const float *>(p.k), *V = static_cast<const float *>(p.v);

  float m[2], l[2], o[2][D / 32];
  int b = g0 < g1 ? find_seq(prefix, p.B, p.Hkv, g0) : 0;
  for (int64_t g = g0; g < g1; ++g) {
    while ((int64_t)p.Hkv * prefix[b + 1] <= g) ++b;
    const int nb = prefix[b + 1] - prefix[b];
    const int64_t r = g - (int64_t)p.Hkv * prefix[b];
    const int kvh = (int)(r / nb), i = (int)(r % nb);
    const int64_t U = (int64_t)p.Hkv * prefix[b] + (int64_t)kvh * nb;
    const int64_t u = (int64_t)b * p.Hkv + kvh;
    const int T = clamp_len(__ldg(p.seq_lens + b), (int)p.t_cap);
    const bool first = i == 0 || g == g0, last = i == nb - 1 || g == g1 - 1;
    const int p0 = i * kF32Tile;
    if (first) {
      const float *q = static_cast<const float *>(p.q) + ((int64_t)b * p.Hkv * p.G + (int64_t)kvh * p.G) * D;
      for (int e = threadIdx.x; e < p.G * D; e += nthr) cp_async_4(smem_u32(Qs + e), q + e);
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        m[hs] = -INFINITY;
        l[hs] = 0.f;
        for (int j = 0; j < D / 32; ++j) o[hs][j] = 0.f;
      }
    }
    // the tile's slots once, then every element of its K and V rows in flight
    // at once (4-byte cp.async into the padded rows)
    for (int rr = threadIdx.x; rr < kF32Tile; rr += nthr) {
      const int pos = p0 + rr;
      const int64_t slot = pos < T ? slot_of(p.page_table, p.max_pages, p.page_size, b, pos) : -1;
      slots[rr] = slot >= 0 && slot < p.num_slots ? slot : -1;
    }
    __syncthreads();
#pragma unroll 8
    for (int e = threadIdx.x; e < kF32Tile * D; e += 32 * kF32Warps) {
      const int rr = e / D, col = e % D;
      const int64_t slot = slots[rr];
      float *kd = Ks + rr * (D + 1) + col, *vd = Vs + rr * (D + 1) + col;
      if (slot >= 0) {
        cp_async_4(smem_u32(kd), K + (slot * p.Hkv + kvh) * D + col);
        cp_async_4(smem_u32(vd), V + (slot * p.Hkv + kvh) * D + col);
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
      const int h = warp + kF32Warps * hs;
      if (h >= p.G) break;
      float s[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int rr = lane + 32 * j;
        float acc = 0.f;
#pragma unroll 4
        for (int e = 0; e < D; ++e) acc = fmaf(Qs[h * D + e], Ks[rr * (D + 1) + e], acc);
        s[j] = p0 + rr < T ? acc : -INFINITY;
        if (p0 + rr < T) p.ws.logits[(u * p.ustride + p0 + rr) * p.G + h] = acc;
      }
      const float mx = warp_max(fmaxf(s[0], s[1]));
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
        for (int rr = 0; rr < kF32Tile; ++rr) {
          const float pp = __shfl_sync(0xffffffffu, pr[rr >> 5], rr & 31);
          acc = fmaf(pp, Vs[rr * (D + 1) + lane + 32 * j], acc);
        }
        o[hs][j] = acc;
      }
    }
    __syncthreads();
    if (last) {
      const int64_t j = blockIdx.x - part.cfirst(U);
      if (j < 0 || j >= p.R) {
        if (threadIdx.x == 0) set_error(p.ws.err, kErrRecord);
        continue;
      }
      float *rec = p.ws.records + (size_t)(u * p.R + j) * p.G * (D + 2);
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        const int h = warp + kF32Warps * hs;
        if (h >= p.G) break;
        if (lane == 0) {
          rec[h] = m[hs];
          rec[p.G + h] = l[hs];
        }
        for (int jj = 0; jj < D / 32; ++jj) rec[2 * p.G + h * D + lane + 32 * jj] = o[hs][jj];
      }
    }
  }
}

template <int D, bool FP8, int NCW, int NSTAGE, int NSL, int NT>
cudaError_t launch_mma_t(const FullParams &p, const CUtensorMap &tmk, const CUtensorMap &tmv, int grid,
                         cudaStream_t s) {
  using C = Cfg<D, FP8, NCW, NSTAGE, NSL, NT>;
  const size_t smem = C::bytes(p.B);
  auto kern = full_attn_mma_kernel<D, FP8, NCW, NSTAGE, NSL, NT>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  return launch_ex(kern, dim3(grid), dim3(32 * (NCW + kProducerWarps<FP8>)), smem, s, 0, tmk, tmv, p);
}

template <int NSTAGE, bool FP8>
cudaError_t launch_tc_t(const FullParams &p, const CUtensorMap &tmk, const CUtensorMap &tmv, int grid,
                        cudaStream_t s) {
  using C = Cfg<128, FP8, 4, NSTAGE, 2, 2, true>;
  const size_t smem = C::bytes(p.B);
  auto kern = full_attn_tc_kernel<NSTAGE, FP8>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  return launch_ex(kern, dim3(grid), dim3(32 * (4 + 1 + kProducerWarps<FP8>)), smem, s, 0, tmk, tmv, p);
}

template <int D, bool FP8, int NCW, int NSTAGE, int NSL, int NT>
cudaError_t launch_fused_t(const FullParams &p, const ScoreParams &sp, const CUtensorMap &tmk,
                           const CUtensorMap &tmv, int grid, cudaStream_t s) {
  using C = Cfg<D, FP8, NCW, NSTAGE, NSL, NT>;
  static_assert(kTailBufOffset + 4 * kTailChunk <= (size_t)C::STAGE * NSTAGE, "score-pass arrays fit in the stages");
  const size_t smem = C::bytes(p.B);
  auto kern = full_attn_fused_kernel<D, FP8, NCW, NSTAGE, NSL, NT>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), (int)smem);
  if (e != cudaSuccess) return e;
  return launch_coop(kern, dim3(grid), dim3(32 * (NCW + kProducerWarps<FP8>)), smem, s, tmk, tmv, p, sp);
}

}  // namespace

size_t full_tc_smem_bytes(int B, bool fp8) {
  return fp8 ? Cfg<128, true, 4, 3, 2, 2, true>::bytes(B) : Cfg<128, false, 4, 3, 2, 2, true>::bytes(B);
}

cudaError_t launch_full_mma(const FullParams &p, const CUtensorMap &tmk, const CUtensorMap &tmv, bool fp8,
                            const FullMmaConfig &cfg, int grid, cudaStream_t s) {
  if (cfg.tc) {  // 3 stages (bf16 with 2: 181 us against 133 at MQA 256K)
    if (!(p.D == 128 && cfg.ncw == 4 && cfg.nstage == 3 && cfg.nsl == 2 && (p.G == 16 || p.G == 32)))
      return cudaErrorInvalidConfiguration;
    return fp8 ? launch_tc_t<3, true>(p, tmk, tmv, grid, s) : launch_tc_t<3, false>(p, tmk, tmv, grid, s);
  }
#define HS2_FULL_CASE(D_, F_, W_, S_, L_, N_)                                                        \
  if (p.D == D_ && fp8 == F_ && cfg.ncw == W_ && cfg.nstage == S_ && cfg.nsl == L_ && cfg.nt == N_) \
    return launch_mma_t<D_, F_, W_, S_, L_, N_>(p, tmk, tmv, grid, s);
  HS2_FULL_CASE(128, false, 8, 3, 1, 1)
  HS2_FULL_CASE(128, false, 4, 6, 1, 1)
  HS2_FULL_CASE(128, false, 4, 3, 2, 1)
  HS2_FULL_CASE(64, false, 8, 6, 1, 1)
  HS2_FULL_CASE(64, false, 4, 6, 1, 1)
  HS2_FULL_CASE(128, true, 8, 3, 2, 1)
  HS2_FULL_CASE(128, true, 6, 4, 2, 1)
  HS2_FULL_CASE(128, true, 4, 6, 2, 1)
  HS2_FULL_CASE(128, true, 16, 3, 1, 1)
  HS2_FULL_CASE(128, true, 12, 4, 1, 1)
  HS2_FULL_CASE(128, true, 8, 6, 1, 1)
  HS2_FULL_CASE(128, true, 4, 8, 1, 1)
  // 16 heads per warp (groups of 16 and 32 query heads)
  HS2_FULL_CASE(128, false, 8, 3, 1, 2)
  HS2_FULL_CASE(128, false, 4, 3, 2, 2)
  HS2_FULL_CASE(64, false, 8, 6, 1, 2)
  HS2_FULL_CASE(128, true, 4, 6, 2, 2)
#undef HS2_FULL_CASE
  return cudaErrorInvalidConfiguration;
}

cudaError_t launch_full_fused(const FullParams &p, const ScoreParams &sp, const CUtensorMap &tmk,
                              const CUtensorMap &tmv, bool fp8, const FullMmaConfig &cfg, int grid, cudaStream_t s) {
  if (cfg.tc) {  // (bf16 only)
    if (!(p.D == 128 && !fp8 && cfg.ncw == 4 && cfg.nstage == 3 && cfg.nsl == 2 && (p.G == 16 || p.G == 32)))
      return cudaErrorInvalidConfiguration;
    using C = Cfg<128, false, 4, 3, 2, 2, true>;
    static_assert(kTailBufOffset + 4 * kTailChunk <= (size_t)C::STAGE * 3, "score-pass arrays fit in the stages");
    const size_t smem = C::bytes(p.B);
    auto kern = full_attn_fused_tc_kernel<3>;
    cudaError_t e = set_smem_once(reinterpret_cast<const void *>(kern), (int)smem);
    if (e != cudaSuccess) return e;
    return launch_coop(kern, dim3(grid), dim3(32 * (4 + 1 + 1)), smem, s, tmk, tmv, p, sp);
  }
#define HS2_FUSED_CASE(D_, F_, W_, S_, L_, N_)                                                       \
  if (p.D == D_ && fp8 == F_ && cfg.ncw == W_ && cfg.nstage == S_ && cfg.nsl == L_ && cfg.nt == N_) \
    return launch_fused_t<D_, F_, W_, S_, L_, N_>(p, sp, tmk, tmv, grid, s);
  // the default configuration of each case
  HS2_FUSED_CASE(128, false, 4, 3, 2, 1)
  HS2_FUSED_CASE(64, false, 8, 6, 1, 1)
  HS2_FUSED_CASE(128, true, 8, 3, 2, 1)
  HS2_FUSED_CASE(128, false, 4, 3, 2, 2)
  HS2_FUSED_CASE(128, true, 4, 6, 2, 2)
#undef HS2_FUSED_CASE
  return cudaErrorInvalidConfiguration;
}

int full_f32_tile() { return kF32Tile; }
int full_f32_ctas_per_sm() { return 2; }

cudaError_t launch_full_f32(const FullParams &p, int grid, cudaStream_t s) {
  const size_t smem = (size_t)(2 * kF32Tile * (p.D + 1) + 8 * p.D) * 4 + kF32Tile * 8 + (size_t)(p.B + 1) * 4;
  cudaError_t e;
  if (p.D == 64) {
    e = set_smem_once(reinterpret_cast<const void *>(full_attn_f32_kernel<64>), (int)smem);
    if (e != cudaSuccess) return e;
    return launch_ex(full_attn_f32_kernel<64>, dim3(grid), dim3(32 * kF32Warps), smem, s, 0, p);
  } else if (p.D == 128) {
    e = set_smem_once(reinterpret_cast<const void *>(full_attn_f32_kernel<128>), (int)smem);
    if (e != cudaSuccess) return e;
    return launch_ex(full_attn_f32_kernel<128>, dim3(grid), dim3(32 * kF32Warps), smem, s, 0, p);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hs2
