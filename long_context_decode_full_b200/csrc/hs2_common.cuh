// hs2_common.cuh -- shared device helpers of libhs2 (sm_100a).
//
// PTX wrappers (mbarrier, TMA bulk-tensor loads, cp.async, ldmatrix,
// mma.sync), the workspace layout and the balanced tile partition that the
// full-attention kernels and the score kernel agree on.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hs2 {

// ---------------------------------------------------------------- constants
constexpr int kHistBins = 4096;          // score histogram: float bits 30..19
constexpr int kHistShift = 19;
constexpr int kScoreThreads = 256;
constexpr int kFinalThreads = 512;
constexpr long long kSpinLimitCycles = 4000000000LL;  // ~2 s at 2 GHz
constexpr int kMaxBatchSmem = 4096;      // sequences whose tile prefix fits in smem
constexpr int kSubRange = 512;           // positions per filter-warp list
constexpr float kBandMargin = 4e-4f;     // relative margin of the selection guard band
constexpr int kMaxSelect = 4096;         // window + k_global upper bound
constexpr int64_t kMaxContext = int64_t(1) << 23;  // positions per sequence
constexpr int kMaxGroup = 32;            // query heads per KV head (MQA: all of them)

// Error bits of the sticky workspace flag.
constexpr uint32_t kErrFullWait = 1u;    // consumer timed out on a full barrier
constexpr uint32_t kErrEmptyWait = 2u;   // producer timed out on an empty barrier
constexpr uint32_t kErrRecord = 4u;      // record index outside its unit's slots

// ---------------------------------------------------------------- workspace
// Every array of the full-attention call lives in the caller's workspace.
struct FullWs {
  uint32_t *err;         // sticky error flag (offset 0 of the workspace)
  int32_t *prefix;       // [B + 1] tiles before sequence b (tile = kernel's TILE positions)
  float *logits;         // [U, t_cap, G] raw q.k per position and head (fp32, unscaled)
  float *records;        // [U, R, G * (D + 2)]: m[G], l[G], o[G][D] of each segment
  float *scores;         // [U, t_cap] group score of the selectable positions
  int32_t *above;        // [U, t_cap] positions above the threshold bin, per 512-position list
  uint2 *cand;           // [U, t_cap] (score bits, position) inside the threshold bin, same lists
  int2 *subcnt;          // [U, nsub] (above, in-bin) counts of each list
  uint32_t *hist;        // [U, kHistBins], then ticket [U] and one spare word [U]
  uint32_t *ticket;      // [U]
  int2 *thr;             // [U] (threshold bin, count strictly above it)
  double *lse;           // [U, kMaxGroup] per-head log-sum-exp of the scaled logits
};

// Balanced partition of the tile space over N persistent CTAs.  Tiles are
// ordered by (sequence, kv head, tile); CTA c owns [c*total/N, (c+1)*total/N).
// A unit (sequence, kv head) is cut into segments, one per CTA that touches
// it; segment j of unit u writes record u*R + j, with j = c - cfirst(U_u).
struct Partition {
  int64_t total;  // Hkv * sum_b n_b
  int32_t N;      // CTAs
  __device__ __forceinline__ int64_t start(int64_t c) const { return c * total / N; }
  // the CTA that owns tile x
  __device__ __forceinline__ int64_t cfirst(int64_t x) const { return ((x + 1) * N - 1) / total; }
  // whether CTA c owns any tile (with more CTAs than tiles some own none,
  // and their record slots are never written)
  __device__ __forceinline__ bool owns_tiles(int64_t c) const { return start(c + 1) > start(c); }
};

// ---------------------------------------------------------------- misc
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void set_error(uint32_t *err, uint32_t bit) {
  if (err) atomicOr(err, bit);
}

__device__ __forceinline__ int clamp_len(int t, int t_cap) { return t < 0 ? 0 : (t > t_cap ? t_cap : t); }

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase with the given parity to complete; gives up after
// `limit` cycles (kSpinLimitCycles by default) and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, long long limit = kSpinLimitCycles) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(a, parity)) {
    if (clock64() - t0 > limit) return false;
  }
  return true;
}
// cp.async completion of this thread's earlier copies arrives on `bar`
// (the barrier's expected count must include this arrival).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------- TMA
// 3-D tiled bulk-tensor load into this CTA's shared memory (no multicast).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint64_t *bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
// The same load with an L2 eviction-priority hint (a createpolicy value).
__device__ __forceinline__ void tma_load_3d_hint(uint32_t dst, const CUtensorMap *map, uint64_t *bar, int x, int y,
                                                 int z, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
// Untiled bulk copy of `bytes` (a multiple of 16) from global memory into
// this CTA's shared memory, both addresses 16-byte aligned, completing on
// `bar` (no multicast).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
// L2 eviction policies.  The logits are read back by the score pass right
// after the attention kernel (evict last), so most of them are still in L2
// then.  Marking the K/V stream (read once) evict-first helps only when the
// logits fit in L2 beside it; with more logits than L2 it slows the stream.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void st_global_hint(float *addr, float a, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(addr), "f"(a), "l"(policy) : "memory");
}
__device__ __forceinline__ void st_global_hint(float *addr, float a, float b, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;" ::"l"(addr), "f"(a), "f"(b), "l"(policy)
               : "memory");
}
// orders this thread's generic-proxy shared-memory accesses before later
// async-proxy (TMA) accesses to the same memory
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- cp.async
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// ---------------------------------------------------------------- ldmatrix / mma
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void lds128(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D(16x8, f32) += A(16x16) * B(16x8); A rows = M, B columns = N.
__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}
// four E4M3 codes (bytes 0..3 of w) -> two f16x2 (exact): lo = bytes 0,1,
// hi = bytes 2,3, the lower byte of each pair in the lower half
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t &lo, uint32_t &hi) {
  asm("{\n\t.reg .b16 a, b;\n\t"
      "mov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Transpose of an 8x8 matrix of 16-bit values held as one fragment (lane
// 4r + c holds row r, columns 2c and 2c+1) into the same fragment layout.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t r;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}

// 128-byte swizzle of a [rows][128 B] panel (the TMA SWIZZLE_128B pattern):
// 16-byte chunk c of row r lives at chunk c ^ (r & 7).
__device__ __forceinline__ uint32_t swz(uint32_t panel, int row, int chunk) {
  return panel + row * 128 + (((chunk ^ row) & 7) << 4);
}

// ---------------------------------------------------------------- PDL
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may be scheduled before its predecessor finishes; it must
// wait before touching anything an earlier kernel produces or consumes.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 2^x by the MUFU approximation (flushes subnormal results to zero)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---------------------------------------------------------------- warp reductions
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace hs2
