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
constexpr int AD_CHUNK = 64;  // keys per CTA (two per lane in the score pass)

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global.L2::128B [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}

// K/V rows of the chunk live in shared memory with a row pitch of D + 8
// elements, so that 32 lanes reading 16 bytes of 32 different rows hit
// distinct banks.
template <int D>
__global__ void __launch_bounds__(AD_THREADS)
attn_decode_kernel(const __grid_constant__ AttnDecParams p) {
  constexpr int PITCH = D + 8;
  constexpr int VPR = D / 8;  // 16-byte vectors per row
  __shared__ __align__(16) bf16 Ks[AD_CHUNK * PITCH];
  __shared__ __align__(16) bf16 Vs[AD_CHUNK * PITCH];
  __shared__ __align__(16) float qs[D];
  __shared__ float ps[AD_CHUNK];
  __shared__ float s_red[AD_WARPS];
  __shared__ float s_o[AD_THREADS / D > 1 ? AD_THREADS / D : 1][D];
  __shared__ int s_last;

  const int bh = blockIdx.x, s = blockIdx.y;
  const int b = bh / p.H, h = bh - b * p.H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long HD = (long long)p.H * D;

  pdl_launch_dependents();
  pdl_wait();

  int pos = p.seqlens[b];
  pos = pos < 0 ? 0 : (pos >= p.S_max ? p.S_max - 1 : pos);
  const int L = pos + 1;
  const int start = s * AD_CHUNK;
  const int n = min(L - start, AD_CHUNK);  // keys in this CTA (may be <= 0)

  float* mypart = p.part + ((long long)bh * p.nsplit + s) * (D + 2);
  if (n > 0) {
    // ---- all K/V rows of the chunk in flight at once ----
    const bf16* kg = p.k_cache + ((long long)b * p.S_max + start) * HD + (long long)h * D;
    const bf16* vg = p.v_cache + ((long long)b * p.S_max + start) * HD + (long long)h * D;
    const bool has_new = p.k_new != nullptr && pos >= start && pos < start + n;
    for (int idx = tid; idx < n * VPR; idx += AD_THREADS) {
      const int j = idx / VPR, c = (idx - j * VPR) * 8;
      if (has_new && start + j == pos) continue;
      cp_async16(Ks + j * PITCH + c, kg + (long long)j * HD + c);
      cp_async16(Vs + j * PITCH + c, vg + (long long)j * HD + c);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    const long long qoff = ((long long)b * p.H + h) * D;
    for (int c = tid; c < D; c += AD_THREADS) qs[c] = bf2f(p.q[qoff + c]) * p.scale_log2;
    if (has_new) {
      // The new key/value: written to the cache and used from shared memory.
      const int j = pos - start;
      const long long goff = ((long long)b * p.S_max + pos) * HD + (long long)h * D;
      for (int c = tid * 8; c < D; c += AD_THREADS * 8) {
        const uint4 kv = *reinterpret_cast<const uint4*>(p.k_new + qoff + c);
        const uint4 vv = *reinterpret_cast<const uint4*>(p.v_new + qoff + c);
        *reinterpret_cast<uint4*>(Ks + j * PITCH + c) = kv;
        *reinterpret_cast<uint4*>(Vs + j * PITCH + c) = vv;
        *reinterpret_cast<uint4*>(p.k_cache + goff + c) = kv;
        *reinterpret_cast<uint4*>(p.v_cache + goff + c) = vv;
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();

    // ---- scores: one key per lane (two lanes' worth per warp pass) ----
    float mloc = -INFINITY;
    for (int j = tid; j < n; j += AD_THREADS) {
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < D; c += 8) {
        const uint4 u = *reinterpret_cast<const uint4*>(Ks + j * PITCH + c);
        const float4 q0 = *reinterpret_cast<const float4*>(qs + c);
        const float4 q1 = *reinterpret_cast<const float4*>(qs + c + 4);
        dot = fmaf(q0.x, bf_lo(u.x), dot); dot = fmaf(q0.y, bf_hi(u.x), dot);
        dot = fmaf(q0.z, bf_lo(u.y), dot); dot = fmaf(q0.w, bf_hi(u.y), dot);
        dot = fmaf(q1.x, bf_lo(u.z), dot); dot = fmaf(q1.y, bf_hi(u.z), dot);
        dot = fmaf(q1.z, bf_lo(u.w), dot); dot = fmaf(q1.w, bf_hi(u.w), dot);
      }
      ps[j] = dot;
      mloc = fmaxf(mloc, dot);
    }
    mloc = warp_max(mloc);
    if (lane == 0) s_red[warp] = mloc;
    __syncthreads();
    float M = s_red[0];
#pragma unroll
    for (int w = 1; w < AD_WARPS; ++w) M = fmaxf(M, s_red[w]);
    __syncthreads();
    float lsum = 0.f;
    for (int j = tid; j < n; j += AD_THREADS) {
      const float e = exp2f(ps[j] - M);
      ps[j] = e;
      lsum += e;
    }
    lsum = warp_sum(lsum);
    if (lane == 0) s_red[warp] = lsum;
    __syncthreads();
    float Lc = 0.f;
#pragma unroll
    for (int w = 0; w < AD_WARPS; ++w) Lc += s_red[w];

    // ---- o = sum_j p_j v_j: thread owns one dimension and a key stripe ----
    constexpr int STRIPES = AD_THREADS / D > 1 ? AD_THREADS / D : 1;
    const int dim = tid % D, stripe = tid / D;
    float o = 0.f;
    if (stripe < STRIPES) {
      for (int j = stripe; j < n; j += STRIPES) o = fmaf(ps[j], bf2f(Vs[j * PITCH + dim]), o);
      s_o[stripe][dim] = o;
    }
    __syncthreads();
    if (tid < D) {
      o = 0.f;
#pragma unroll
      for (int st = 0; st < STRIPES; ++st) o += s_o[st][tid];
      if (p.nsplit == 1) {
        p.out[((long long)b * p.H + h) * D + tid] = f2bf(o / Lc);
        return;
      }
      __stcg(mypart + 2 + tid, o);
      if (tid == 0) { __stcg(mypart, M); __stcg(mypart + 1, Lc); }
    }
  } else {
    // Empty slice (beyond the current length): a neutral partial.
    for (int dd = tid; dd < D; dd += AD_THREADS) __stcg(mypart + 2 + dd, 0.f);
    if (tid == 0) { __stcg(mypart, -INFINITY); __stcg(mypart + 1, 0.f); }
  }
  if (p.nsplit == 1) return;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(p.counters + bh, 1) == p.nsplit - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // Merge the split partials: per-split weights exp2(M_s - M) computed once
  // into shared memory, then every thread sums its dimension over splits
  // with independent loads (fixed split order: deterministic).
  const float* base = p.part + (long long)bh * p.nsplit * (D + 2);
  float* wts = ps;  // AD_CHUNK floats, reused (nsplit <= 1024 handled in passes)
  float Mg = -INFINITY;
  for (int sp = tid; sp < p.nsplit; sp += AD_THREADS) Mg = fmaxf(Mg, __ldcg(base + (long long)sp * (D + 2)));
  Mg = warp_max(Mg);
  if (lane == 0) s_red[warp] = Mg;
  __syncthreads();
  Mg = s_red[0];
#pragma unroll
  for (int w = 1; w < AD_WARPS; ++w) Mg = fmaxf(Mg, s_red[w]);
  __syncthreads();
  float Lg = 0.f, acc = 0.f;
  for (int s0 = 0; s0 < p.nsplit; s0 += AD_CHUNK) {
    const int ns = min(AD_CHUNK, p.nsplit - s0);
    if (tid < ns) {
      const float ms = __ldcg(base + (long long)(s0 + tid) * (D + 2));
      const float w = (ms == -INFINITY) ? 0.f : exp2f(ms - Mg);
      wts[tid] = w;
      Lg += w * __ldcg(base + (long long)(s0 + tid) * (D + 2) + 1);
    }
    __syncthreads();
    if (tid < D) {
      const float* ob = base + (long long)s0 * (D + 2) + 2 + tid;
      int sp = 0;
      for (; sp + 4 <= ns; sp += 4) {
        const float o0 = __ldcg(ob + (long long)sp * (D + 2));
        const float o1 = __ldcg(ob + (long long)(sp + 1) * (D + 2));
        const float o2 = __ldcg(ob + (long long)(sp + 2) * (D + 2));
        const float o3 = __ldcg(ob + (long long)(sp + 3) * (D + 2));
        acc += (o0 * wts[sp] + o1 * wts[sp + 1]) + (o2 * wts[sp + 2] + o3 * wts[sp + 3]);
      }
      for (; sp < ns; ++sp) acc += __ldcg(ob + (long long)sp * (D + 2)) * wts[sp];
    }
    __syncthreads();
  }
  Lg = warp_sum(Lg);
  if (lane == 0) s_red[warp] = Lg;
  __syncthreads();
  Lg = 0.f;
#pragma unroll
  for (int w = 0; w < AD_WARPS; ++w) Lg += s_red[w];
  if (tid < D) p.out[((long long)b * p.H + h) * D + tid] = f2bf(acc / Lg);
  if (tid == 0) p.counters[bh] = 0;
}

}  // namespace

int attn_decode_launch(AttnDecParams p, int target_ctas, cudaStream_t stream) {
  (void)target_ctas;
  const int pairs = p.B * p.H;
  p.chunk = AD_CHUNK;
  p.nsplit = ceil_div(p.S_max, AD_CHUNK);
  if (p.nsplit > 1024) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  const dim3 grid(pairs, p.nsplit);
  // History K and V once (cache length is only known on the device; the
  // tag counts the full capacity), plus q, out and the new rows.
  const LaunchTag tag{"attn_decode", 2.0 * 2.0 * pairs * (double)p.S_max * p.D, 0.0};
  if (p.D == 128) return launch_pdl(tag, attn_decode_kernel<128>, grid, dim3(AD_THREADS), 0, stream, p);
  if (p.D == 64) return launch_pdl(tag, attn_decode_kernel<64>, grid, dim3(AD_THREADS), 0, stream, p);
  return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace fsvd
