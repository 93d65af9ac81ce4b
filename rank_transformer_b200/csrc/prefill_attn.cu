// Full-sequence attention for prefill (causal) and the encoder
// (bidirectional): one CTA per (64-query tile, batch*head), four warps of 16
// query rows, K/V streamed through a double-buffered shared-memory ring in
// 64-key blocks with an online softmax in fp32 (exp2 domain).  The two
// contractions (Q K^T and P V) run on the warp-level bf16 tensor-core MMA
// (m16n8k16) fed by ldmatrix from 128-byte-swizzled shared memory.
//
// FlashSVD v1.5 (gist.science explainer), Technical Summary, Methodology 2:
// prefill keeps its own full-sequence attention; the K/V it attends over are
// the rows the prefill projections wrote into the dense KV cache.
#include "kernels.h"

namespace fsvd {

namespace {

constexpr int BQ = 64, BKV = 64, AP_THREADS = 128;

__device__ __forceinline__ void cp_async16_zfill(void* smem, const void* gmem, bool valid) {
  const uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sa), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t* r, const void* p) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, const void* p) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Element offset of (row, 16-byte chunk) in a [rows x D] tile whose chunks
// are XOR-swizzled by row, so that ldmatrix row addresses hit distinct banks.
template <int D>
__device__ __forceinline__ int swz(int row, int chunk) {
  return row * D + ((chunk ^ (row & 7)) << 3);
}

template <int D>
__device__ __forceinline__ void load_tile(bf16* dst, const bf16* src, long long row_stride, int row0,
                                          int rows_valid) {
  constexpr int CH = D / 8;
  for (int idx = threadIdx.x; idx < 64 * CH; idx += AP_THREADS) {
    const int r = idx / CH, c = idx - r * CH;
    const bool ok = row0 + r < rows_valid;
    const bf16* g = src + (ok ? (long long)(row0 + r) * row_stride + c * 8 : 0);
    cp_async16_zfill(dst + swz<D>(r, c), g, ok);
  }
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(AP_THREADS)
attn_prefill_kernel(const __grid_constant__ AttnPfParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  bf16* Qs = reinterpret_cast<bf16*>(sm);
  bf16* Ks = Qs + BQ * D;         // [2][BKV][D]
  bf16* Vs = Ks + 2 * BKV * D;    // [2][BKV][D]

  const int nqt = gridDim.x;
  const int qt = CAUSAL ? nqt - 1 - blockIdx.x : blockIdx.x;  // heavy tiles first
  const int bh = blockIdx.y, b = bh / p.H, h = bh - b * p.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = qt * BQ;
  const long long HD = (long long)p.H * D;
  const bf16* qg = p.q + ((long long)b * p.S) * HD + (long long)h * D;
  const bf16* kg = p.k + ((long long)b * p.S_max) * HD + (long long)h * D;
  const bf16* vg = p.v + ((long long)b * p.S_max) * HD + (long long)h * D;

  pdl_launch_dependents();
  pdl_wait();

  const int kv_end = CAUSAL ? min(p.S, q0 + BQ) : p.S;
  const int nblocks = (kv_end + BKV - 1) / BKV;

  load_tile<D>(Qs, qg, HD, q0, p.S);
  load_tile<D>(Ks, kg, HD, 0, p.S);
  load_tile<D>(Vs, vg, HD, 0, p.S);
  asm volatile("cp.async.commit_group;" ::: "memory");

  uint32_t qf[D / 16][4];
  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  const int g = lane >> 2, t4 = lane & 3;
  const int row_a = q0 + warp * 16 + g;  // absolute query rows of this thread
  const int row_b = row_a + 8;

  for (int j = 0; j < nblocks; ++j) {
    if (j + 1 < nblocks) {
      const int nb = (j + 1) & 1;
      load_tile<D>(Ks + nb * BKV * D, kg, HD, (j + 1) * BKV, p.S);
      load_tile<D>(Vs + nb * BKV * D, vg, HD, (j + 1) * BKV, p.S);
      asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    if (j == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = kk * 2 + (lane >> 4);
        ldsm_x4(qf[kk], Qs + swz<D>(r, c));
      }
    }
    const bf16* Kb = Ks + (j & 1) * BKV * D;
    const bf16* Vb = Vs + (j & 1) * BKV * D;

    // ---- S = Q K^T : 16 x 64 per warp ----
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int n2 = 0; n2 < 4; ++n2) {  // pairs of 8-key tiles
        uint32_t kf[4];
        const int r = n2 * 16 + (lane & 7) + (lane >> 4) * 8;
        const int c = kk * 2 + ((lane >> 3) & 1);
        ldsm_x4(kf, Kb + swz<D>(r, c));
        mma16816(s[2 * n2], qf[kk], kf[0], kf[1]);
        mma16816(s[2 * n2 + 1], qf[kk], kf[2], kf[3]);
      }
    }

    // ---- online softmax (rows row_a, row_b) ----
    const int k0 = j * BKV;
    float mx[2] = {m_r[0], m_r[1]};
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = k0 + n * 8 + 2 * t4 + (e & 1);
        const int row = (e < 2) ? row_a : row_b;
        float v = s[n][e] * p.scale_log2;
        if (key >= p.S || (CAUSAL && key > row)) v = -INFINITY;
        s[n][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
    }
    float corr[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      corr[i] = (m_r[i] == -INFINITY) ? 0.f : exp2f(m_r[i] - mx[i]);
      m_r[i] = mx[i];
      l_r[i] *= corr[i];
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      o[n][0] *= corr[0]; o[n][1] *= corr[0];
      o[n][2] *= corr[1]; o[n][3] *= corr[1];
    }
    uint32_t pf[4][4];  // P as the A operand of P V, four 16-key steps
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const float p0 = (mx[0] == -INFINITY) ? 0.f : exp2f(s[n][0] - mx[0]);
      const float p1 = (mx[0] == -INFINITY) ? 0.f : exp2f(s[n][1] - mx[0]);
      const float p2 = (mx[1] == -INFINITY) ? 0.f : exp2f(s[n][2] - mx[1]);
      const float p3 = (mx[1] == -INFINITY) ? 0.f : exp2f(s[n][3] - mx[1]);
      l_r[0] += p0 + p1;
      l_r[1] += p2 + p3;
      const int ks = n >> 1, hi = n & 1;
      pf[ks][hi * 2 + 0] = pack_bf2(p0, p1);
      pf[ks][hi * 2 + 1] = pack_bf2(p2, p3);
    }

    // ---- O += P V ----
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
      for (int n2 = 0; n2 < D / 16; ++n2) {
        uint32_t vf[4];
        const int r = ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = n2 * 2 + (lane >> 4);
        ldsm_x4_t(vf, Vb + swz<D>(r, c));
        mma16816(o[2 * n2], pf[ks], vf[0], vf[1]);
        mma16816(o[2 * n2 + 1], pf[ks], vf[2], vf[3]);
      }
    }
    __syncthreads();
  }

  // ---- normalise and store ----
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 1);
    l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 2);
  }
  const float inv_a = l_r[0] > 0.f ? 1.f / l_r[0] : 0.f;
  const float inv_b = l_r[1] > 0.f ? 1.f / l_r[1] : 0.f;
  bf16* og = p.out + ((long long)b * p.S) * HD + (long long)h * D;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int col = n * 8 + 2 * t4;
    if (row_a < p.S)
      *reinterpret_cast<uint32_t*>(og + (long long)row_a * HD + col) = pack_bf2(o[n][0] * inv_a, o[n][1] * inv_a);
    if (row_b < p.S)
      *reinterpret_cast<uint32_t*>(og + (long long)row_b * HD + col) = pack_bf2(o[n][2] * inv_b, o[n][3] * inv_b);
  }
}

template <int D, bool CAUSAL>
int launch_attn(const AttnPfParams& p, cudaStream_t stream) {
  auto kern = attn_prefill_kernel<D, CAUSAL>;
  constexpr int SMEM = (BQ * D + 4 * BKV * D) * 2;
  static bool configured = false;
  if (!configured) {
    FSVD_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM));
    configured = true;
  }
  const dim3 grid(ceil_div(p.S, BQ), p.B * p.H);
  const double S = p.S, HD = (double)p.H * D;
  const double flops = 4.0 * p.B * p.H * S * S * D * (CAUSAL ? 0.5 : 1.0);
  const LaunchTag tag{CAUSAL ? "attn_prefill_causal" : "attn_prefill_bidir",
                      2.0 * 4.0 * p.B * S * HD, flops};
  return launch_pdl(tag, kern, grid, dim3(AP_THREADS), (size_t)SMEM, stream, p);
}

}  // namespace

int attn_prefill_launch(const AttnPfParams& p, cudaStream_t stream) {
  // tcgen05 kernel (attn_tc.cu) for every shape it covers; this mma.sync
  // kernel remains for the rest
  const int st = attn_prefill_tc_launch(p, stream);
  if (st != FLASHSVD_ERR_UNSUPPORTED_SHAPE && st != FLASHSVD_ERR_NOT_INITIALIZED) return st;
  if (p.D == 128) return p.causal ? launch_attn<128, true>(p, stream) : launch_attn<128, false>(p, stream);
  if (p.D == 64) return p.causal ? launch_attn<64, true>(p, stream) : launch_attn<64, false>(p, stream);
  return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace fsvd
