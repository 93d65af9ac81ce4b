// Row-wise glue around the factorized linears: RMSNorm, LayerNorm, rotary
// table, embedding gather, greedy pick and sequence-length advance.  All
// are memory-bound one-pass kernels with 16-byte vector access.
#include "kernels.h"

namespace fsvd {

namespace {

constexpr int NT = 256;

__device__ __forceinline__ float block_sum(float v, float* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += sh[w];
  return t;
}

__device__ __forceinline__ void ld8(const bf16* p, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  v[0] = bf_lo(u.x); v[1] = bf_hi(u.x); v[2] = bf_lo(u.y); v[3] = bf_hi(u.y);
  v[4] = bf_lo(u.z); v[5] = bf_hi(u.z); v[6] = bf_lo(u.w); v[7] = bf_hi(u.w);
}
__device__ __forceinline__ void unpack8(const uint4& u, float* v) {
  v[0] = bf_lo(u.x); v[1] = bf_hi(u.x); v[2] = bf_lo(u.y); v[3] = bf_hi(u.y);
  v[4] = bf_lo(u.z); v[5] = bf_hi(u.z); v[6] = bf_lo(u.w); v[7] = bf_hi(u.w);
}
__device__ __forceinline__ void st8(bf16* p, const float* v) {
  uint4 u;
  u.x = pack_bf2(v[0], v[1]); u.y = pack_bf2(v[2], v[3]);
  u.z = pack_bf2(v[4], v[5]); u.w = pack_bf2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p) = u;
}

// Rows of up to ROW_VEC * 8 * blockDim.x elements (8192 at 256 threads) are
// held in registers; the launcher gives rows of up to 4096 elements 128
// threads, so that every row of a 2048-row norm is resident in one wave
// (16 CTAs per SM).  The gains (and LayerNorm's bias) do not depend on the
// previous kernel: they are loaded before the programmatic-launch wait.
constexpr int ROW_VEC = 4;  // 16-byte vectors per thread

__global__ void __launch_bounds__(NT)
rmsnorm_kernel(const bf16* x, const bf16* g, bf16* y, int d, float eps) {
  __shared__ float sh[NT / 32];
  pdl_launch_dependents();
  const int nt = blockDim.x;
  // x and g stay packed (bf16) in registers between the two passes
  uint4 graw[ROW_VEC], xraw[ROW_VEC];
#pragma unroll
  for (int i = 0; i < ROW_VEC; ++i) {
    const int c = (threadIdx.x + i * nt) * 8;
    if (c < d) graw[i] = *reinterpret_cast<const uint4*>(g + c);
  }
  pdl_wait();
  const long long row = blockIdx.x;
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < ROW_VEC; ++i) {
    const int c = (threadIdx.x + i * nt) * 8;
    if (c < d) {
      xraw[i] = *reinterpret_cast<const uint4*>(x + row * d + c);
      float v[8];
      unpack8(xraw[i], v);
#pragma unroll
      for (int j = 0; j < 8; ++j) ss = fmaf(v[j], v[j], ss);
    }
  }
  const float rs = rsqrtf(block_sum(ss, sh) / (float)d + eps);
#pragma unroll
  for (int i = 0; i < ROW_VEC; ++i) {
    const int c = (threadIdx.x + i * nt) * 8;
    if (c < d) {
      float v[8], gg[8], o[8];
      unpack8(xraw[i], v);
      unpack8(graw[i], gg);
#pragma unroll
      for (int j = 0; j < 8; ++j) o[j] = v[j] * rs * gg[j];
      st8(y + row * d + c, o);
    }
  }
}

__global__ void __launch_bounds__(NT)
layernorm_kernel(const bf16* x, const bf16* g, const bf16* b, bf16* y, int d,
                 float eps) {
  __shared__ float sh[NT / 32];
  pdl_launch_dependents();
  const int nt = blockDim.x;
  uint4 graw[ROW_VEC], braw[ROW_VEC], xraw[ROW_VEC];
#pragma unroll
  for (int i = 0; i < ROW_VEC; ++i) {
    const int c = (threadIdx.x + i * nt) * 8;
    if (c < d) {
      graw[i] = *reinterpret_cast<const uint4*>(g + c);
      braw[i] = *reinterpret_cast<const uint4*>(b + c);
    }
  }
  pdl_wait();
  const long long row = blockIdx.x;
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < ROW_VEC; ++i) {
    const int c = (threadIdx.x + i * nt) * 8;
    if (c < d) {
      xraw[i] = *reinterpret_cast<const uint4*>(x + row * d + c);
      float v[8];
      unpack8(xraw[i], v);
#pragma unroll
      for (int j = 0; j < 8; ++j) s += v[j];
    }
  }
  const float mean = block_sum(s, sh) / (float)d;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < ROW_VEC; ++i) {
    const int c = (threadIdx.x + i * nt) * 8;
    if (c < d) {
      float v[8];
      unpack8(xraw[i], v);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float t = v[j] - mean;
        q = fmaf(t, t, q);
      }
    }
  }
  const float rs = rsqrtf(block_sum(q, sh) / (float)d + eps);
#pragma unroll
  for (int i = 0; i < ROW_VEC; ++i) {
    const int c = (threadIdx.x + i * nt) * 8;
    if (c < d) {
      float v[8], gg[8], bb[8], o[8];
      unpack8(xraw[i], v);
      unpack8(graw[i], gg);
      unpack8(braw[i], bb);
#pragma unroll
      for (int j = 0; j < 8; ++j) o[j] = (v[j] - mean) * rs * gg[j] + bb[j];
      st8(y + row * d + c, o);
    }
  }
}

__global__ void rope_table_kernel(float* cs, float* sn, int S_max, int D,
                                  double base) {
  pdl_launch_dependents();
  pdl_wait();
  const int half = D / 2;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)S_max * half) return;
  const int p = (int)(idx / half), i = (int)(idx - (long long)p * half);
  const double ang = (double)p * pow(base, -2.0 * (double)i / (double)D);
  cs[idx] = (float)cos(ang);
  sn[idx] = (float)sin(ang);
}

__global__ void __launch_bounds__(NT)
embed_kernel(const int* tokens, const bf16* emb, bf16* x, int d, int vocab) {
  pdl_launch_dependents();
  pdl_wait();
  int t = tokens[blockIdx.x];
  t = t < 0 ? 0 : (t >= vocab ? vocab - 1 : t);
  const uint4* src = reinterpret_cast<const uint4*>(emb + (long long)t * d);
  uint4* dst = reinterpret_cast<uint4*>(x + (long long)blockIdx.x * d);
  for (int c = threadIdx.x; c < d / 8; c += NT) dst[c] = src[c];
}

__global__ void __launch_bounds__(1024)
greedy_kernel(const float* logits, int* next, int vocab) {
  __shared__ float sv[32];
  __shared__ int si[32];
  pdl_launch_dependents();
  pdl_wait();
  const float* row = logits + (long long)blockIdx.x * vocab;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  // GR_UNROLL independent loads in flight per thread (one at a time would
  // leave the row's read bound by the load latency, ~30 in a row per thread
  // at a 32000-entry vocabulary)
  constexpr int GR_UNROLL = 16;
  const int stride = blockDim.x;
  for (int j0 = threadIdx.x; j0 < vocab; j0 += stride * GR_UNROLL) {
    float v[GR_UNROLL];
#pragma unroll
    for (int u = 0; u < GR_UNROLL; ++u) {
      const int j = j0 + u * stride;
      v[u] = j < vocab ? __ldg(row + j) : -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < GR_UNROLL; ++u)
      if (v[u] > bv) { bv = v[u]; bi = j0 + u * stride; }  // j increases: ties keep the lower index
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) { sv[warp] = bv; si[warp] = bi; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
      if (sv[w] > bv || (sv[w] == bv && si[w] < bi)) { bv = sv[w]; bi = si[w]; }
    next[blockIdx.x] = bi == 0x7fffffff ? 0 : bi;
  }
}

__global__ void advance_kernel(int* seqlens, int B) {
  pdl_launch_dependents();
  pdl_wait();
  for (int b = threadIdx.x; b < B; b += blockDim.x) seqlens[b] += 1;
}

// Rows of up to 2048 elements: one warp per row (VPL 16-byte vectors per
// lane), eight rows per CTA, no CTA barriers.
constexpr int WR_ROWS = 8;

template <int VPL, bool LN>
__global__ void __launch_bounds__(WR_ROWS * 32)
norm_warp_kernel(const bf16* x, const bf16* g, const bf16* b, bf16* y, int M, int d, float eps) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * WR_ROWS + (threadIdx.x >> 5);
  if (row >= M) return;
  float v[VPL][8];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int c = (lane + i * 32) * 8;
    if (c < d) {
      ld8(x + row * d + c, v[i]);
#pragma unroll
      for (int j = 0; j < 8; ++j) s = LN ? s + v[i][j] : fmaf(v[i][j], v[i][j], s);
    }
  }
  s = warp_sum(s);
  float mean = 0.f, rs;
  if (LN) {
    mean = s / (float)d;
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if ((lane + i * 32) * 8 < d)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float t = v[i][j] - mean;
          q = fmaf(t, t, q);
        }
    rs = rsqrtf(warp_sum(q) / (float)d + eps);
  } else {
    rs = rsqrtf(s / (float)d + eps);
  }
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int c = (lane + i * 32) * 8;
    if (c < d) {
      float gg[8], bb[8], o[8];
      ld8(g + c, gg);
      if (LN) ld8(b + c, bb);
#pragma unroll
      for (int j = 0; j < 8; ++j) o[j] = LN ? (v[i][j] - mean) * rs * gg[j] + bb[j] : v[i][j] * rs * gg[j];
      st8(y + row * d + c, o);
    }
  }
}

// Threads of the one-CTA-per-row norms: 128 up to 4096 elements, else NT.
inline int norm_threads(int d) { return d <= 128 * ROW_VEC * 8 ? 128 : NT; }

template <bool LN>
int norm_warp_launch(const bf16* x, const bf16* g, const bf16* b, bf16* y, int M, int d, float eps,
                     cudaStream_t s) {
  const LaunchTag tag{LN ? "layernorm" : "rmsnorm", 4.0 * M * d, 0.0};
  const dim3 grid(ceil_div(M, WR_ROWS)), block(WR_ROWS * 32);
  switch (ceil_div(d, 256)) {
    case 1: return launch_pdl(tag, norm_warp_kernel<1, LN>, grid, block, 0, s, x, g, b, y, M, d, eps);
    case 2: return launch_pdl(tag, norm_warp_kernel<2, LN>, grid, block, 0, s, x, g, b, y, M, d, eps);
    case 3: return launch_pdl(tag, norm_warp_kernel<3, LN>, grid, block, 0, s, x, g, b, y, M, d, eps);
    case 4: return launch_pdl(tag, norm_warp_kernel<4, LN>, grid, block, 0, s, x, g, b, y, M, d, eps);
    case 5: case 6: return launch_pdl(tag, norm_warp_kernel<6, LN>, grid, block, 0, s, x, g, b, y, M, d, eps);
    default: return launch_pdl(tag, norm_warp_kernel<8, LN>, grid, block, 0, s, x, g, b, y, M, d, eps);
  }
}

}  // namespace

int rmsnorm_launch(const bf16* x, const bf16* g, bf16* y, int M, int d,
                   float eps, cudaStream_t s) {
  if (d > NT * ROW_VEC * 8) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return FLASHSVD_OK;
  if (d <= 2048) return norm_warp_launch<false>(x, g, nullptr, y, M, d, eps, s);
  return launch_pdl(LaunchTag{"rmsnorm", 4.0 * M * d, 0.0}, rmsnorm_kernel, dim3(M), dim3(norm_threads(d)), 0, s,
                    x, g, y, d, eps);
}

int layernorm_launch(const bf16* x, const bf16* g, const bf16* b, bf16* y,
                     int M, int d, float eps, cudaStream_t s) {
  if (d > NT * ROW_VEC * 8) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return FLASHSVD_OK;
  if (d <= 2048) return norm_warp_launch<true>(x, g, b, y, M, d, eps, s);
  return launch_pdl(LaunchTag{"layernorm", 4.0 * M * d, 0.0}, layernorm_kernel, dim3(M), dim3(norm_threads(d)), 0,
                    s, x, g, b, y, d, eps);
}

int rope_table_launch(float* c, float* sn, int S_max, int D, float base,
                      cudaStream_t s) {
  const long long n = (long long)S_max * (D / 2);
  if (n == 0) return FLASHSVD_OK;
  return launch_pdl(LaunchTag{"rope_table", 8.0 * n, 0.0}, rope_table_kernel, dim3((unsigned)((n + NT - 1) / NT)), dim3(NT), 0, s,
                    c, sn, S_max, D, (double)base);
}

int embed_launch(const int* tokens, const bf16* emb, bf16* x, int B, int d,
                 int vocab, cudaStream_t s) {
  if (B == 0) return FLASHSVD_OK;
  return launch_pdl(LaunchTag{"embed", 4.0 * B * d, 0.0}, embed_kernel, dim3(B), dim3(NT), 0, s, tokens, emb, x, d, vocab);
}

int greedy_launch(const float* logits, int* next, int M, int vocab,
                  cudaStream_t s) {
  if (M == 0) return FLASHSVD_OK;
  return launch_pdl(LaunchTag{"greedy", 4.0 * M * vocab, 0.0}, greedy_kernel, dim3(M), dim3(1024), 0, s, logits, next, vocab);
}

int advance_launch(int* seqlens, int B, cudaStream_t s) {
  return launch_pdl(LaunchTag{"advance", 8.0 * B, 0.0}, advance_kernel, dim3(1), dim3(32), 0, s, seqlens, B);
}

}  // namespace fsvd
