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
#include "hs2_warp_attn.cuh"

namespace hs2 {

namespace {

struct StageMeta {
  int32_t b, kvh, tile, flags;
  int32_t rec, T, pad0, pad1;
};
constexpr int kFirst = 1, kLast = 2, kDone = 4;

template <int D, bool FP8, int NCW, int NSTAGE, int NSL, int NT>
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
  static constexpr size_t OFF_PREFIX = OFF_META + NSTAGE * sizeof(StageMeta);
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

// The attention pass of one CTA; with FUSED the CTA then runs the score pass
// of the selection (hs2_fused_tail.cuh) over the tiles it attended.
template <int D, bool FP8, int NCW, int NSTAGE, int NSL, int NT, bool FUSED>
__device__ __forceinline__ void full_attn_body(const CUtensorMap &tmk, const CUtensorMap &tmv, const FullParams &p,
                                               const ScoreParams *sp) {
  using C = Cfg<D, FP8, NCW, NSTAGE, NSL, NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  uint64_t *empty = full + NSTAGE;
  uint64_t *cbar = empty + NSTAGE;  // consumer-warp rendezvous at segment ends
  StageMeta *meta = reinterpret_cast<StageMeta *>(smem + C::OFF_META);
  int32_t *prefix = reinterpret_cast<int32_t *>(smem + C::OFF_PREFIX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool producer = warp >= NCW;
  const bool tma_role = warp == NCW;  // the other producer warp (E4M3) gathers scales

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], FP8 ? 33u : 1u);
      mbar_init(&empty[s], (uint32_t)NCW);
    }
    mbar_init(cbar, (uint32_t)NCW);
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
  } else if (!producer) {
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
  int32_t *prefix = reinterpret_cast<int32_t *>(Qs + 8 * D);
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
      for (int e = threadIdx.x; e < p.G * D; e += nthr) Qs[e] = q[e];
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        m[hs] = -INFINITY;
        l[hs] = 0.f;
        for (int j = 0; j < D / 32; ++j) o[hs][j] = 0.f;
      }
    }
    for (int e = threadIdx.x; e < kF32Tile * D; e += nthr) {
      const int rr = e / D, col = e % D, pos = p0 + rr;
      float kv = 0.f, vv = 0.f;
      const int64_t slot = pos < T ? slot_of(p.page_table, p.max_pages, p.page_size, b, pos) : -1;
      if (slot >= 0 && slot < p.num_slots) {
        kv = K[(slot * p.Hkv + kvh) * D + col];
        vv = V[(slot * p.Hkv + kvh) * D + col];
      }
      Ks[rr * (D + 1) + col] = kv;
      Vs[rr * (D + 1) + col] = vv;
    }
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
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_ex(kern, dim3(grid), dim3(32 * (NCW + kProducerWarps<FP8>)), smem, s, 0, tmk, tmv, p);
}

template <int D, bool FP8, int NCW, int NSTAGE, int NSL, int NT>
cudaError_t launch_fused_t(const FullParams &p, const ScoreParams &sp, const CUtensorMap &tmk,
                           const CUtensorMap &tmv, int grid, cudaStream_t s) {
  using C = Cfg<D, FP8, NCW, NSTAGE, NSL, NT>;
  static_assert(kTailBufOffset + 4 * kTailChunk <= (size_t)C::STAGE * NSTAGE, "score-pass arrays fit in the stages");
  const size_t smem = C::bytes(p.B);
  auto kern = full_attn_fused_kernel<D, FP8, NCW, NSTAGE, NSL, NT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_coop(kern, dim3(grid), dim3(32 * (NCW + kProducerWarps<FP8>)), smem, s, tmk, tmv, p, sp);
}

}  // namespace

cudaError_t launch_full_mma(const FullParams &p, const CUtensorMap &tmk, const CUtensorMap &tmv, bool fp8,
                            const FullMmaConfig &cfg, int grid, cudaStream_t s) {
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
  const size_t smem = (size_t)(2 * kF32Tile * (p.D + 1) + 8 * p.D) * 4 + (size_t)(p.B + 1) * 4;
  cudaError_t e;
  if (p.D == 64) {
    e = cudaFuncSetAttribute(full_attn_f32_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_ex(full_attn_f32_kernel<64>, dim3(grid), dim3(32 * kF32Warps), smem, s, 0, p);
  } else if (p.D == 128) {
    e = cudaFuncSetAttribute(full_attn_f32_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_ex(full_attn_f32_kernel<128>, dim3(grid), dim3(32 * kF32Warps), smem, s, 0, p);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hs2
