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
// One kernel, bound by reading the two weight matrices once.  A CTA takes 128
// output columns, one split of 128 rows of W and up to 8 tokens:
//   - each lane owns 4 columns and issues its warp's 16 row loads (8 bytes
//     each, 256 bytes per warp and row) before any arithmetic, so about 32 KB
//     per CTA is in flight;
//   - the 8 warps' partial sums meet in shared memory and the CTA's tile of
//     partial sums goes to the workspace;
//   - the last CTA of each (K or V, column tile, token group) to finish -- a
//     ticket counter in the workspace -- adds the splits' tiles: 8 / (tokens)
//     warps per token, each a fixed share of the splits in split order, then
//     the shares in warp order (so the result does not depend on which CTA
//     came last), stores the rows
//     (E4M3: one warp per token holds a whole head of 128 columns, so the
//     row max is a warp reduction) and resets its ticket to zero.
#include "hs2.h"
#include "hs2_internal.h"

namespace hs2 {

namespace {

constexpr int kBridgeCols = 128;    // output columns per CTA, 4 per lane
constexpr int kBridgeRows = 128;    // rows of W per CTA (one split)
constexpr int kBridgeTokens = 8;    // tokens per CTA
constexpr int kBridgeThreads = 256;
constexpr int kBridgeWarps = kBridgeThreads / 32;
constexpr int kRowsPerWarp = kBridgeRows / kBridgeWarps;
static_assert(kBridgeTokens == kBridgeWarps, "the final sums give one warp to each token");
static_assert(kBridgeCols == 4 * 32, "a lane owns 4 columns");

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t u) {
  __nv_bfloat162 v;
  memcpy(&v, &u, 4);
  return __bfloat1622float2(v);  // .x is the lower address
}

// TOK token slots per CTA (1, 2, 4 or 8: the batch rounded up to a power of
// two, 8 above 4), so a small batch does not pay for 8 tokens' FMAs.
template <int TOK>
__global__ void __launch_bounds__(kBridgeThreads) bridge_kernel(const BridgeParams p) {
  static_assert(TOK >= 1 && TOK <= kBridgeTokens, "token slots");
  __shared__ float sh_h[TOK][kBridgeRows];                                 // the tokens' hidden slice
  __shared__ __align__(16) float sh_red[kBridgeWarps][TOK][kBridgeCols];   // per-warp partial sums
  __shared__ int sh_last;
  griddep_wait();
  griddep_launch_dependents();
  const int tile = blockIdx.x, split = blockIdx.y;
  const int kv = blockIdx.z & 1, grp = blockIdx.z >> 1, b0 = grp * kBridgeTokens;
  const int nb = min(kBridgeTokens, p.B - b0);
  const int r0 = split * kBridgeRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int col = tile * kBridgeCols + 4 * lane;
  const bool active = col < p.N;  // N is a multiple of 64: a lane's 4 columns are all in or all out

  // the weight rows first (they are the traffic), then the hidden slice
  const __nv_bfloat16 *w = kv ? p.wv : p.wk;
  uint2 wr[kRowsPerWarp];
#pragma unroll
  for (int j = 0; j < kRowsPerWarp; ++j) {
    const int r = r0 + warp + j * kBridgeWarps;
    wr[j] = active ? __ldg(reinterpret_cast<const uint2 *>(w + (int64_t)r * p.N + col)) : make_uint2(0u, 0u);
  }
  for (int e = threadIdx.x; e < TOK * kBridgeRows; e += kBridgeThreads) {
    const int t = e / kBridgeRows, r = e % kBridgeRows;
    sh_h[t][r] = t < nb ? __bfloat162float(p.h[(int64_t)(b0 + t) * p.d_model + r0 + r]) : 0.f;
  }
  __syncthreads();

  float acc[TOK][4];
#pragma unroll
  for (int t = 0; t < TOK; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
#pragma unroll
  for (int j = 0; j < kRowsPerWarp; ++j) {
    const int r = warp + j * kBridgeWarps;
    const float2 w01 = bf16x2_to_float2(wr[j].x), w23 = bf16x2_to_float2(wr[j].y);
#pragma unroll
    for (int t = 0; t < TOK; ++t) {
      const float hv = sh_h[t][r];
      acc[t][0] = fmaf(hv, w01.x, acc[t][0]);
      acc[t][1] = fmaf(hv, w01.y, acc[t][1]);
      acc[t][2] = fmaf(hv, w23.x, acc[t][2]);
      acc[t][3] = fmaf(hv, w23.y, acc[t][3]);
    }
  }
#pragma unroll
  for (int t = 0; t < TOK; ++t)
    *reinterpret_cast<float4 *>(&sh_red[warp][t][4 * lane]) = make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]);
  __syncthreads();

  // this split's tile: warp `tok` sums the 8 warps' rows of token tok in warp order
  const int tok = warp;
  if (tok < nb && active) {
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w8 = 0; w8 < kBridgeWarps; ++w8) s = add4(s, *reinterpret_cast<const float4 *>(&sh_red[w8][tok][4 * lane]));
    __stcg(reinterpret_cast<float4 *>(p.partial + (((int64_t)kv * p.nsplit + split) * p.B + b0 + tok) * p.N + col), s);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // one gpu-scope fence after the barrier orders every thread's partial
    // store (fences are cumulative) before the ticket
    __threadfence();
    int *ticket = p.tickets + ((int64_t)kv * p.ntiles + tile) * p.ngroups + grp;
    const int last = atomicAdd(ticket, 1) == p.nsplit - 1;
    if (last) *ticket = 0;  // every split has counted: ready for the next call
    sh_last = last;
  }
  __syncthreads();
  if (!sh_last) return;
  __threadfence();

  // last CTA: the splits of token t are read by the warps t * wpt .. (t + 1)
  // * wpt - 1 at once, each a fixed share of the splits in split order (one
  // round of loads), and the shares are then added in warp order: the result
  // does not depend on timing
  const int wpt = kBridgeWarps / nb;  // warps per token
  {
    const int t = warp / wpt, k = warp % wpt;
    float4 x4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t < nb && active) {
      const int s0 = k * p.nsplit / wpt, s1 = (k + 1) * p.nsplit / wpt;
      const float *src = p.partial + ((int64_t)kv * p.nsplit * p.B + b0 + t) * p.N + col;
      const int64_t step = (int64_t)p.B * p.N;
#pragma unroll 16
      for (int sp = s0; sp < s1; ++sp) x4 = add4(x4, __ldcg(reinterpret_cast<const float4 *>(src + sp * step)));
    }
    *reinterpret_cast<float4 *>(&sh_red[warp][0][4 * lane]) = x4;
  }
  __syncthreads();
  if (tok >= nb) return;
  const int b = b0 + tok;
  float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k = 0; k < wpt; ++k) x = add4(x, *reinterpret_cast<const float4 *>(&sh_red[tok * wpt + k][0][4 * lane]));
  const int T = clamp_len(__ldg(p.seq_lens + b), (int)p.t_cap);
  if (T < 1) return;  // no token to append
  const int64_t pos = T - 1;
  const int64_t slot = p.page_table == nullptr
                           ? (int64_t)b * p.page_size + pos
                           : (int64_t)__ldg(p.page_table + (int64_t)b * p.max_pages + pos / p.page_size) *
                                     p.page_size + pos % p.page_size;
  if (slot < 0 || slot >= p.num_slots) return;  // a page outside the cache: nothing is written
  const int kvh = col / p.D, d = col % p.D;      // a lane's 4 columns share one head
  const int64_t e = (slot * p.Hkv + kvh) * p.D + d;
  void *cache = kv ? p.v : p.k;
  if (p.kv_dtype == HS2_BF16) {
    if (!active) return;
    const __nv_bfloat162 lo = __floats2bfloat162_rn(x.x, x.y), hi = __floats2bfloat162_rn(x.z, x.w);
    uint2 u;
    memcpy(&u.x, &lo, 4);
    memcpy(&u.y, &hi, 4);
    *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(cache) + e) = u;
  } else if (p.kv_dtype == HS2_F32) {
    if (!active) return;
    *reinterpret_cast<float4 *>(static_cast<float *>(cache) + e) = x;
  } else {
    // E4M3 caches have D = 128 = kBridgeCols: the warp holds head kvh of token
    // b whole, every lane active.  scale = max|x| / 448, codes nearest-even,
    // saturated.
    const float amax = warp_max(fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
    const float scale = amax > 0.f ? amax / 448.f : 1.f;
    const __nv_fp8_e4m3 c0(x.x / scale), c1(x.y / scale), c2(x.z / scale), c3(x.w / scale);
    const uint32_t packed = (uint32_t)c0.__x | ((uint32_t)c1.__x << 8) | ((uint32_t)c2.__x << 16) |
                            ((uint32_t)c3.__x << 24);
    *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(cache) + e) = packed;
    if (lane == 0) (kv ? p.v_scale : p.k_scale)[slot * p.Hkv + kvh] = scale;
  }
}

int ticket_words(int B, int N) {
  return 2 * ((N + kBridgeCols - 1) / kBridgeCols) * ((B + kBridgeTokens - 1) / kBridgeTokens);
}

size_t align256_(size_t n) { return (n + 255) & ~size_t(255); }

}  // namespace

int bridge_splits(int d_model) { return d_model / kBridgeRows; }
int bridge_row_multiple() { return kBridgeRows; }

size_t bridge_workspace_bytes(int B, int d_model, int N) {
  return align256_((size_t)ticket_words(B, N) * 4) + align256_((size_t)2 * bridge_splits(d_model) * B * N * 4);
}

cudaError_t launch_bridge(const BridgeParams &p0, void *workspace, cudaStream_t s) {
  BridgeParams p = p0;
  p.ntiles = (p.N + kBridgeCols - 1) / kBridgeCols;
  p.ngroups = (p.B + kBridgeTokens - 1) / kBridgeTokens;
  p.tickets = static_cast<int32_t *>(workspace);
  p.partial = reinterpret_cast<float *>(static_cast<char *>(workspace) + align256_((size_t)ticket_words(p.B, p.N) * 4));
  const dim3 grid(p.ntiles, p.nsplit, 2 * p.ngroups);
  const dim3 block(kBridgeThreads);
  if (p.B == 1) return launch_ex(bridge_kernel<1>, grid, block, 0, s, 0, p);
  if (p.B == 2) return launch_ex(bridge_kernel<2>, grid, block, 0, s, 0, p);
  if (p.B <= 4) return launch_ex(bridge_kernel<4>, grid, block, 0, s, 0, p);
  return launch_ex(bridge_kernel<kBridgeTokens>, grid, block, 0, s, 0, p);
}

}  // namespace hs2
