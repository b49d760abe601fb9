// hs2_bridge.cu -- KV Bridging append of one decode step (HySparse2
// announcement, "KV Bridging" paragraphs: each Cross-Decoder full-attention
// layer builds its own KV cache from the input hidden state of the matching
// Self-Decoder full-attention layer, through its own K and V projections).
//
// For every sequence b the new token's rows are k_b = h_b W_k and
// v_b = h_b W_v (h [d_model] bf16, W [d_model, Hkv * d] bf16, fp32
// accumulation), written at position T_b - 1 of the paged cache: bf16 or fp32
// as computed, or E4M3 with one fp32 scale per (token, kv head) = max|x| / 448.
//
// Two kernels, both memory- or latency-bound (the weights are read once):
//   gemv  -- split-K over the hidden dimension: a CTA takes 64 output columns,
//            256 rows of W and up to 8 tokens; each lane reads a bf16 pair of
//            every row (128 B per warp, coalesced), the warps' partial sums
//            meet in shared memory and land in the workspace;
//   store -- one CTA per (sequence, kv head, K or V): the splits' partial
//            sums in a fixed order (deterministic), then the row is stored
//            (E4M3: block max, scale, codes rounded to nearest even with
//            saturation).
#include "hs2.h"
#include "hs2_internal.h"

namespace hs2 {

namespace {

constexpr int kBridgeCols = 64;     // output columns per gemv CTA
constexpr int kBridgeRows = 256;    // rows of W per gemv CTA (one split)
constexpr int kBridgeTokens = 8;    // tokens per gemv CTA
constexpr int kBridgeThreads = 256;
constexpr int kBridgeWarps = kBridgeThreads / 32;

__global__ void __launch_bounds__(kBridgeThreads) bridge_gemv_kernel(const BridgeParams p) {
  __shared__ float sh_h[kBridgeTokens][kBridgeRows];                     // the tokens' hidden slice
  __shared__ float sh_red[kBridgeWarps][kBridgeTokens][kBridgeCols];     // per-warp partial sums
  griddep_wait();
  griddep_launch_dependents();
  const int tile = blockIdx.x, split = blockIdx.y;
  const int kv = blockIdx.z & 1, b0 = (blockIdx.z >> 1) * kBridgeTokens;
  const int nb = min(kBridgeTokens, p.B - b0);
  const int r0 = split * kBridgeRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < kBridgeTokens * kBridgeRows; e += blockDim.x) {
    const int t = e / kBridgeRows, r = e % kBridgeRows;
    sh_h[t][r] = t < nb ? __bfloat162float(p.h[(int64_t)(b0 + t) * p.d_model + r0 + r]) : 0.f;
  }
  __syncthreads();
  const __nv_bfloat16 *w = kv ? p.wv : p.wk;
  const int col = tile * kBridgeCols + 2 * lane;
  float acc[kBridgeTokens][2];
#pragma unroll
  for (int t = 0; t < kBridgeTokens; ++t) acc[t][0] = acc[t][1] = 0.f;
#pragma unroll 4
  for (int r = warp; r < kBridgeRows; r += kBridgeWarps) {
    const __nv_bfloat162 w2 =
        __ldg(reinterpret_cast<const __nv_bfloat162 *>(w + (int64_t)(r0 + r) * p.N + col));
    const float2 wf = __bfloat1622float2(w2);
#pragma unroll
    for (int t = 0; t < kBridgeTokens; ++t) {
      const float hv = sh_h[t][r];
      acc[t][0] = fmaf(hv, wf.x, acc[t][0]);
      acc[t][1] = fmaf(hv, wf.y, acc[t][1]);
    }
  }
#pragma unroll
  for (int t = 0; t < kBridgeTokens; ++t) {
    sh_red[warp][t][2 * lane] = acc[t][0];
    sh_red[warp][t][2 * lane + 1] = acc[t][1];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kBridgeTokens * kBridgeCols; e += blockDim.x) {
    const int t = e / kBridgeCols, c = e % kBridgeCols;
    if (t >= nb) continue;
    float s = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < kBridgeWarps; ++w8) s += sh_red[w8][t][c];  // fixed order
    p.partial[(((int64_t)kv * p.nsplit + split) * p.B + b0 + t) * p.N + tile * kBridgeCols + c] = s;
  }
}

__global__ void bridge_store_kernel(const BridgeParams p) {
  __shared__ float sh_max[32];
  griddep_wait();
  griddep_launch_dependents();
  const int b = blockIdx.x, kvh = blockIdx.y, kv = blockIdx.z;
  const int T = clamp_len(__ldg(p.seq_lens + b), (int)p.t_cap);
  if (T < 1) return;  // no token to append
  const int64_t pos = T - 1;
  const int64_t slot = p.page_table == nullptr
                           ? (int64_t)b * p.page_size + pos
                           : (int64_t)__ldg(p.page_table + (int64_t)b * p.max_pages + pos / p.page_size) *
                                     p.page_size + pos % p.page_size;
  if (slot < 0 || slot >= p.num_slots) return;  // a page outside the cache: nothing is written
  const int d = threadIdx.x;                     // blockDim.x = head_dim
  const int n = kvh * p.D + d;
  float x = 0.f;
  for (int s = 0; s < p.nsplit; ++s) x += __ldcg(p.partial + (((int64_t)kv * p.nsplit + s) * p.B + b) * p.N + n);
  const int64_t e = (slot * p.Hkv + kvh) * p.D + d;
  void *cache = kv ? p.v : p.k;
  if (p.kv_dtype == HS2_BF16) {
    static_cast<__nv_bfloat16 *>(cache)[e] = __float2bfloat16_rn(x);
  } else if (p.kv_dtype == HS2_F32) {
    static_cast<float *>(cache)[e] = x;
  } else {  // E4M3: scale = max|x| / 448 over the row, codes nearest-even, saturated
    float m = warp_max(fabsf(x));
    if ((threadIdx.x & 31) == 0) sh_max[threadIdx.x >> 5] = m;
    __syncthreads();
    float amax = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) amax = fmaxf(amax, sh_max[w]);
    const float scale = amax > 0.f ? amax / 448.f : 1.f;
    static_cast<__nv_fp8_e4m3 *>(cache)[e] = __nv_fp8_e4m3(x / scale);
    if (d == 0) (kv ? p.v_scale : p.k_scale)[slot * p.Hkv + kvh] = scale;
  }
}

}  // namespace

int bridge_splits(int d_model) { return d_model / kBridgeRows; }
int bridge_row_multiple() { return kBridgeRows; }

cudaError_t launch_bridge(const BridgeParams &p, cudaStream_t s) {
  const dim3 g1(p.N / kBridgeCols, p.nsplit, 2 * ((p.B + kBridgeTokens - 1) / kBridgeTokens));
  cudaError_t e = launch_ex(bridge_gemv_kernel, g1, dim3(kBridgeThreads), 0, s, 0, p);
  if (e != cudaSuccess) return e;
  return launch_ex(bridge_store_kernel, dim3(p.B, p.Hkv, 2), dim3(p.D), 0, s, 0, p);
}

}  // namespace hs2
