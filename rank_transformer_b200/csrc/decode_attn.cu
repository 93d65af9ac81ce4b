// Dense contiguous-KV decode attention with split-sequence partials.
//
// FlashSVD v1.5 (gist.science explainer), Technical Summary, Methodology 2
// ("reconstruct the present, read the past contiguously"): the history is
// read from a dense [B, S_max, H, D] bf16 cache along one path.  Here each
// (batch, head) pair is split over CTAs along the sequence; every CTA
// streams its slice of K and V once (8 keys per warp in flight) with an
// online softmax in fp32, the CTA's four warps are merged in shared memory,
// and the last CTA of the pair (atomic counter, no waiting) merges the
// split partials in split order, so the result is deterministic.
#include "kernels.h"

namespace fsvd {

namespace {

constexpr int AD_THREADS = 128;
constexpr int AD_WARPS = AD_THREADS / 32;
constexpr int AD_KB = 8;  // keys per warp per batch

template <int EPL>
__device__ __forceinline__ void load_row(const bf16* p, float* v) {
  if (EPL == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    v[0] = bf_lo(u.x); v[1] = bf_hi(u.x); v[2] = bf_lo(u.y); v[3] = bf_hi(u.y);
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    v[0] = bf_lo(u); v[1] = bf_hi(u);
  }
}

template <int EPL>
__device__ __forceinline__ void store_row(bf16* p, const float* v) {
  if (EPL == 4) {
    uint2 u;
    u.x = pack_bf2(v[0], v[1]);
    u.y = pack_bf2(v[2], v[3]);
    *reinterpret_cast<uint2*>(p) = u;
  } else {
    *reinterpret_cast<uint32_t*>(p) = pack_bf2(v[0], v[1]);
  }
}

template <int D>
__global__ void __launch_bounds__(AD_THREADS)
attn_decode_kernel(const __grid_constant__ AttnDecParams p) {
  constexpr int EPL = D / 32;
  __shared__ float s_m[AD_WARPS], s_l[AD_WARPS];
  __shared__ float s_o[AD_WARPS][D];
  __shared__ int s_last;

  const int bh = blockIdx.x, s = blockIdx.y;
  const int b = bh / p.H, h = bh - b * p.H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  pdl_launch_dependents();
  pdl_wait();

  int pos = p.seqlens[b];
  pos = pos < 0 ? 0 : (pos >= p.S_max ? p.S_max - 1 : pos);
  const int L = pos + 1;
  const int start = s * p.chunk;
  const int end = min(L, start + p.chunk);

  const long long HD = (long long)p.H * D;
  const long long head_off = ((long long)b * p.H + h) * D + lane * EPL;
  float qv[EPL];
  load_row<EPL>(p.q + head_off, qv);
#pragma unroll
  for (int e = 0; e < EPL; ++e) qv[e] *= p.scale_log2;

  const bf16* kbase = p.k_cache + (long long)b * p.S_max * HD + (long long)h * D + lane * EPL;
  const bf16* vbase = p.v_cache + (long long)b * p.S_max * HD + (long long)h * D + lane * EPL;

  // The CTA whose slice holds the current position writes the new key and
  // value into the cache and uses them directly (no other CTA reads them).
  const bool has_new = p.k_new != nullptr && pos >= start && pos < end;
  float kn[EPL], vn[EPL];
  if (has_new) {
    load_row<EPL>(p.k_new + head_off, kn);
    load_row<EPL>(p.v_new + head_off, vn);
    if (warp == 0) {
      store_row<EPL>(p.k_cache + ((long long)b * p.S_max + pos) * HD + (long long)h * D + lane * EPL, kn);
      store_row<EPL>(p.v_cache + ((long long)b * p.S_max + pos) * HD + (long long)h * D + lane * EPL, vn);
    }
  }

  float m = -INFINITY, l = 0.f, acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;

  for (int j0 = start + warp * AD_KB; j0 < end; j0 += AD_WARPS * AD_KB) {
    float kv[AD_KB][EPL], vv[AD_KB][EPL];
#pragma unroll
    for (int i = 0; i < AD_KB; ++i) {
      const int j = j0 + i;
      if (j < end) {
        if (has_new && j == pos) {
#pragma unroll
          for (int e = 0; e < EPL; ++e) { kv[i][e] = kn[e]; vv[i][e] = vn[e]; }
        } else {
          load_row<EPL>(kbase + (long long)j * HD, kv[i]);
          load_row<EPL>(vbase + (long long)j * HD, vv[i]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < EPL; ++e) { kv[i][e] = 0.f; vv[i][e] = 0.f; }
      }
    }
    float sc[AD_KB];
    float mb = -INFINITY;
#pragma unroll
    for (int i = 0; i < AD_KB; ++i) {
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) dot = fmaf(qv[e], kv[i][e], dot);
      dot = warp_sum(dot);
      sc[i] = (j0 + i < end) ? dot : -INFINITY;
      mb = fmaxf(mb, sc[i]);
    }
    const float mn = fmaxf(m, mb);
    const float corr = exp2f(m - mn);
    l *= corr;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] *= corr;
#pragma unroll
    for (int i = 0; i < AD_KB; ++i) {
      const float pe = exp2f(sc[i] - mn);
      l += pe;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[e] = fmaf(pe, vv[i][e], acc[e]);
    }
    m = mn;
  }

  // ---- merge the warps of this CTA ----
  if (lane == 0) { s_m[warp] = m; s_l[warp] = l; }
#pragma unroll
  for (int e = 0; e < EPL; ++e) s_o[warp][lane * EPL + e] = acc[e];
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < AD_WARPS; ++w) M = fmaxf(M, s_m[w]);
  float Lc = 0.f;
  float wgt[AD_WARPS];
#pragma unroll
  for (int w = 0; w < AD_WARPS; ++w) {
    wgt[w] = (M == -INFINITY) ? 0.f : exp2f(s_m[w] - M);
    Lc += s_l[w] * wgt[w];
  }

  if (p.nsplit == 1) {
    for (int dd = tid; dd < D; dd += AD_THREADS) {
      float o = 0.f;
#pragma unroll
      for (int w = 0; w < AD_WARPS; ++w) o += s_o[w][dd] * wgt[w];
      p.out[((long long)b * p.H + h) * D + dd] = f2bf(o / Lc);
    }
    return;
  }

  float* mypart = p.part + ((long long)bh * p.nsplit + s) * (D + 2);
  for (int dd = tid; dd < D; dd += AD_THREADS) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < AD_WARPS; ++w) o += s_o[w][dd] * wgt[w];
    __stcg(mypart + 2 + dd, o);
  }
  if (tid == 0) { __stcg(mypart, M); __stcg(mypart + 1, Lc); }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(p.counters + bh, 1) == p.nsplit - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  const float* base = p.part + (long long)bh * p.nsplit * (D + 2);
  float Mg = -INFINITY;
  for (int sp = 0; sp < p.nsplit; ++sp) Mg = fmaxf(Mg, __ldcg(base + sp * (D + 2)));
  float Lg = 0.f;
  for (int sp = 0; sp < p.nsplit; ++sp) {
    const float ms = __ldcg(base + sp * (D + 2));
    if (ms != -INFINITY) Lg += __ldcg(base + sp * (D + 2) + 1) * exp2f(ms - Mg);
  }
  for (int dd = tid; dd < D; dd += AD_THREADS) {
    float o = 0.f;
    for (int sp = 0; sp < p.nsplit; ++sp) {
      const float ms = __ldcg(base + sp * (D + 2));
      if (ms != -INFINITY) o += __ldcg(base + sp * (D + 2) + 2 + dd) * exp2f(ms - Mg);
    }
    p.out[((long long)b * p.H + h) * D + dd] = f2bf(o / Lg);
  }
  if (tid == 0) p.counters[bh] = 0;
}

}  // namespace

int attn_decode_launch(AttnDecParams p, int target_ctas, cudaStream_t stream) {
  const int pairs = p.B * p.H;
  int nsplit = target_ctas / pairs;
  const int max_split = ceil_div(p.S_max, 64);
  nsplit = nsplit < 1 ? 1 : (nsplit > max_split ? max_split : nsplit);
  nsplit = nsplit > 64 ? 64 : nsplit;
  p.chunk = round_up(ceil_div(p.S_max, nsplit), AD_WARPS * AD_KB);
  p.nsplit = ceil_div(p.S_max, p.chunk);
  const dim3 grid(pairs, p.nsplit);
  if (p.D == 128) return launch_pdl(attn_decode_kernel<128>, grid, dim3(AD_THREADS), 0, stream, p);
  if (p.D == 64) return launch_pdl(attn_decode_kernel<64>, grid, dim3(AD_THREADS), 0, stream, p);
  return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace fsvd
