// Decode-regime (M <= 32 rows) factorized linear: split-K GEMV kernels.
//
// FlashSVD v1.5 (gist.science explainer), Technical Summary, Problem
// Statement: decode is memory-bound, so each stage of y = (x U) V is a
// stream over one factor matrix.  One launch handles one stage for up to
// three factor matrices that share the same activation rows:
//   stage 1:  z[m, :]  = A[m, :] . U        (A = x, optionally RMS-normalised)
//   stage 2:  y[m, :]  = z[m, :] . V        (+ fused epilogue)
// The grid is (column tiles x K splits).  Each CTA streams a [KC x 64]
// block of the factor with 16-byte loads (no L1 allocation), multiplies it
// by the matching activation slice held in shared memory (fp32), reduces
// over its 8 warps and writes a partial tile; the last CTA to finish a
// column tile (atomic counter, no waiting) sums the partials in split order
// -- deterministic -- and applies the epilogue.  The intermediate z stays
// in fp32 in a small L2-resident workspace.
#include <cstdio>

#include "kernels.h"

namespace fsvd {

namespace {

constexpr int GV_THREADS = 256;

__device__ __forceinline__ void unpack8(const uint4& v, float* w) {
  w[0] = bf_lo(v.x); w[1] = bf_hi(v.x); w[2] = bf_lo(v.y); w[3] = bf_hi(v.y);
  w[4] = bf_lo(v.z); w[5] = bf_hi(v.z); w[6] = bf_lo(v.w); w[7] = bf_hi(v.w);
}

// (a0, a1) += x * (y0, y1): one packed fp32x2 FMA (sm_100).
__device__ __forceinline__ void gv_ffma2(float& a0, float& a1, float x, float y0, float y1) {
  asm("{\n\t.reg .b64 acc, xx, yy;\n\t"
      "mov.b64 acc, {%0, %1};\n\t"
      "mov.b64 xx, {%2, %2};\n\t"
      "mov.b64 yy, {%3, %4};\n\t"
      "fma.rn.f32x2 acc, xx, yy, acc;\n\t"
      "mov.b64 {%0, %1}, acc;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(x), "f"(y0), "f"(y1));
}

// Split partial stride: the MT x 64 tile plus 8 floats (RMSNORM: the
// split's sums of squares of its rows).
template <int MT>
__host__ __device__ constexpr int gv_part_stride() { return MT * 64 + 8; }

// Global output column of tile column c (0..63) for the column map.
template <int MAP>
__device__ __forceinline__ int tile_col(int t, int c, int D) {
  if (MAP == MAP_PLAIN) return t * 64 + c;
  if (MAP == MAP_ROPE) {
    const int tph = D >> 6, h = t / tph, j = t - h * tph;
    return h * D + j * 32 + (c & 31) + (c >> 5) * (D >> 1);
  }
  return t * 32 + (c & 31);  // SWIGLU: c < 32 gate, c >= 32 up, same column
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t sa = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global.L2::128B [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <int MT, int PRO, int EPI, int MAP>
__global__ void __launch_bounds__(GV_THREADS)
gemv_splitk_kernel(const __grid_constant__ GvParams p) {
  constexpr int NSEG = (MAP == MAP_SWIGLU) ? 2 : 1;
  extern __shared__ __align__(16) float sm[];
  float* As = sm;                                   // [NSEG][MT][KC] fp32
  float* red = As + NSEG * MT * p.KC;               // [8][MT][64] fp32
  bf16* Ws = reinterpret_cast<bf16*>(red + 8 * MT * 64);  // [KC][64] bf16
  __shared__ float s_ssq[MT];  // RMSNORM: sums of squares of this CTA's row slices, then of whole rows
  __shared__ int s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cg = tid & 7, rr = tid >> 3;
  const int tile = blockIdx.x, split = blockIdx.y;
  // row group blockIdx.z: rows m0 .. m0 + Mg - 1 of the launch's p.M rows
  const int m0 = p.m0 + blockIdx.z * MT;
  const int Mg = min(MT, p.M - blockIdx.z * MT);
  const long long slot = (long long)blockIdx.z * gridDim.x + tile;  // partials / counter of this tile

  int pi = 0;
#pragma unroll
  for (int i = 1; i < 3; ++i)
    if (i < p.nprob && tile >= p.tile_start[i]) pi = i;
  const GvProblem P = p.prob[pi];
  const int t = tile - p.tile_start[pi];
  const int hi = cg >> 2;
  const int col = tile_col<MAP>(t, cg * 8, p.D);
  const long long wrow = (MAP == MAP_SWIGLU && hi) ? P.w_row2 : 0;
  const bool colok = col < P.N;
  const int k0 = split * p.KC;
  const int kn = min(p.K - k0, p.KC);
  const int niter = (kn + 31) >> 5;  // <= KC/32

  pdl_launch_dependents();

  // The whole [kn x 64] factor block of this CTA is copied into shared
  // memory with asynchronous 16-byte copies issued before waiting for the
  // previous kernel: factors never depend on it, so these bytes stream
  // while that kernel drains.
  if (colok) {
    const bf16* wp = P.W + (wrow + k0 + rr) * P.ldw + col;
    for (int i = 0; i < niter; ++i) {
      const int kk = rr + 32 * i;
      if (kk < kn) cp_async16(Ws + kk * 64 + cg * 8, wp + (long long)(32 * i) * P.ldw);
    }
  }
  cp_async_commit();

  pdl_wait();
  // ---- stage the activation slice A[m0+m, acol + k0 .. + KC) in fp32 ----
  // RMSNorm: the staged slice holds x * g; the squares of x are summed
  // over this CTA's slice here and over the splits by the reducer, which
  // scales the finished tile by rstd (no pass over the whole row per CTA).
  float ss_t[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) ss_t[m] = 0.f;
  {
    const int kc8 = p.KC >> 3;
    const int items = NSEG * MT * kc8;
    for (int it = tid; it < items; it += GV_THREADS) {
      const int seg = it / (MT * kc8);
      const int rem = it - seg * MT * kc8;
      const int m = rem / kc8;
      const int kk = (rem - m * kc8) * 8;
      float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (m < Mg && kk < kn) {
        const int acol = (seg ? P.a_col2 : P.a_col) + k0 + kk;
        const long long row = m0 + m;
        if (PRO == PRO_F32) {
          const float4* src = reinterpret_cast<const float4*>(p.a32 + row * p.lda + acol);
          const float4 u0 = src[0], u1 = src[1];
          a[0] = u0.x; a[1] = u0.y; a[2] = u0.z; a[3] = u0.w;
          a[4] = u1.x; a[5] = u1.y; a[6] = u1.z; a[7] = u1.w;
        } else {
          unpack8(*reinterpret_cast<const uint4*>(p.x + row * p.ldx + acol), a);
          if (PRO == PRO_RMSNORM) {
            float g[8], ss = 0.f;
            unpack8(*reinterpret_cast<const uint4*>(p.norm_g + acol), g);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              ss = fmaf(a[j], a[j], ss);
              a[j] *= g[j];
            }
#pragma unroll
            for (int mm = 0; mm < MT; ++mm)
              if (mm == m) ss_t[mm] += ss;
          }
        }
      }
      float4* dst = reinterpret_cast<float4*>(As + (seg * MT + m) * p.KC + kk);
      dst[0] = make_float4(a[0], a[1], a[2], a[3]);
      dst[1] = make_float4(a[4], a[5], a[6], a[7]);
    }
  }
  if (PRO == PRO_RMSNORM) {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float ss = warp_sum(ss_t[m]);
      if (lane == 0) red[warp * MT + m] = ss;
    }
  }
  __syncthreads();
  if (PRO == PRO_RMSNORM && tid < MT) {
    float ss = 0.f;
#pragma unroll
    for (int w = 0; w < GV_THREADS / 32; ++w) ss += red[w * MT + tid];
    s_ssq[tid] = ss;  // (red is next written after the barrier below)
  }

  // ---- multiply-accumulate from shared memory ----
  cp_async_wait_all();
  __syncthreads();
  float acc[MT][8];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[m][j] = 0.f;

  const float* Aseg = As + (NSEG == 2 ? hi : 0) * MT * p.KC;
#pragma unroll 4
  for (int i = 0; i < niter; ++i) {
    const int kk = rr + 32 * i;
    if (kk < kn) {
      float w[8];
      unpack8(*reinterpret_cast<const uint4*>(Ws + kk * 64 + cg * 8), w);
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const float a = Aseg[m * p.KC + kk];
#pragma unroll
        for (int j = 0; j < 8; j += 2) gv_ffma2(acc[m][j], acc[m][j + 1], a, w[j], w[j + 1]);
      }
    }
  }

  // ---- reduce the 32 row lanes: 4 per warp by shuffles, 8 warps in smem ----
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float v = acc[m][j];
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      acc[m][j] = v;
    }
  if (lane < 8) {
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int j = 0; j < 8; ++j) red[(warp * MT + m) * 64 + lane * 8 + j] = acc[m][j];
  }
  __syncthreads();

  constexpr int NOUT = MT * 64;
  constexpr int PER = (NOUT + GV_THREADS - 1) / GV_THREADS;
  float val[PER];
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int o = tid + q * GV_THREADS;
    float s = 0.f;
    if (o < NOUT) {
      const int m = o >> 6, c = o & 63;
#pragma unroll
      for (int w = 0; w < GV_THREADS / 32; ++w) s += red[(w * MT + m) * 64 + c];
    }
    val[q] = s;
  }

  if (p.splits > 1) {
    constexpr int NP = gv_part_stride<MT>();
    float* mypart = p.part + (slot * p.splits + split) * NP;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int o = tid + q * GV_THREADS;
      if (o < NOUT) __stcg(mypart + o, val[q]);
    }
    if (PRO == PRO_RMSNORM && tid < MT) __stcg(mypart + NOUT + tid, s_ssq[tid]);
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(p.counters + slot, 1) == p.splits - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // Sum the split partials: LPO threads per output, each a fixed stride
    // of splits, combined by a fixed shuffle tree (deterministic order).
    const float* tp = p.part + slot * p.splits * NP;
    constexpr int LPO = NOUT >= GV_THREADS ? 1 : GV_THREADS / NOUT;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int o = (LPO == 1) ? tid + q * GV_THREADS : tid / LPO;
      const int sub = (LPO == 1) ? 0 : tid % LPO;
      float s = 0.f;
      if (o < NOUT) {
        int sp = sub;
        for (; sp + 3 * LPO < p.splits; sp += 4 * LPO) {
          const float v0 = __ldcg(tp + (long long)sp * NP + o);
          const float v1 = __ldcg(tp + (long long)(sp + LPO) * NP + o);
          const float v2 = __ldcg(tp + (long long)(sp + 2 * LPO) * NP + o);
          const float v3 = __ldcg(tp + (long long)(sp + 3 * LPO) * NP + o);
          s += ((v0 + v1) + (v2 + v3));
        }
        for (; sp < p.splits; sp += LPO) s += __ldcg(tp + (long long)sp * NP + o);
      }
#pragma unroll
      for (int w = 1; w < LPO; w <<= 1) s += __shfl_xor_sync(0xffffffffu, s, w);
      val[q] = s;
    }
    if (PRO == PRO_RMSNORM && tid < MT) {
      float ss = 0.f;  // sums of squares of the whole rows, in split order
      for (int sp = 0; sp < p.splits; ++sp) ss += __ldcg(tp + (long long)sp * NP + NOUT + tid);
      s_ssq[tid] = ss;
    }
    if (tid == 0) p.counters[slot] = 0;  // ready for the next launch
  }

  // ---- epilogue on the finished [MT x 64] tile ----
  __syncthreads();  // red is reused as the finished tile
  float* fin = red;
  {
    constexpr int LPO = NOUT >= GV_THREADS ? 1 : GV_THREADS / NOUT;
    const bool reduced_layout = p.splits > 1 && LPO > 1;
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int o = reduced_layout ? tid / LPO : tid + q * GV_THREADS;
      const bool writer = reduced_layout ? (tid % LPO) == 0 : true;
      if (o < NOUT && writer) fin[o] = val[q];
    }
  }
  __syncthreads();

  if (EPI == EPI_F32 || EPI == EPI_BF16) {
    for (int o = tid; o < NOUT; o += GV_THREADS) {
      const int m = o >> 6, c = o & 63;
      const int gc = tile_col<MAP>(t, c, p.D);
      if (m >= Mg || gc >= P.N) continue;
      const long long row = m0 + m;
      float v = fin[o];
      if (PRO == PRO_RMSNORM) v *= rsqrtf(s_ssq[m] / (float)p.K + p.eps);
      if (EPI == EPI_F32) {
        p.out32[row * p.ldo32 + P.out_col + gc] = v;
      } else {
        if (p.bias) v += bf2f(p.bias[gc]);
        if (p.resid) v += bf2f(p.resid[row * p.ldr + gc]);
        p.out16[row * p.ldo16 + gc] = f2bf(v);
      }
    }
  } else if (EPI == EPI_QKV) {
    const int half = p.D >> 1;
    for (int o = tid; o < MT * 32; o += GV_THREADS) {
      const int m = o >> 5, c = o & 31;
      if (m >= Mg) continue;
      const int b = m0 + m;
      int pos = p.seqlens[b];
      pos = pos < 0 ? 0 : (pos >= p.S_max ? p.S_max - 1 : pos);
      const int glo = tile_col<MAP>(t, c, p.D);
      const int i = glo % p.D;  // rotation index in [0, D/2)
      float lo = fin[m * 64 + c], hv = fin[m * 64 + c + 32];
      if (P.kind < 2) {
        const float cs = p.rope_cos[(long long)pos * half + i];
        const float sn = p.rope_sin[(long long)pos * half + i];
        const float l2 = lo * cs - hv * sn;
        hv = hv * cs + lo * sn;
        lo = l2;
      }
      bf16* dst;
      if (P.kind == 0) dst = p.out16 + (long long)b * p.ldo16;
      else dst = (P.kind == 1 ? p.k_cache : p.v_cache) + ((long long)b * p.S_max + pos) * p.HD;
      dst[glo] = f2bf(lo);
      dst[glo + half] = f2bf(hv);
    }
  } else {  // EPI_SWIGLU
    for (int o = tid; o < MT * 32; o += GV_THREADS) {
      const int m = o >> 5, c = o & 31;
      const int fc = t * 32 + c;
      if (m >= Mg || fc >= P.N) continue;
      const float g = fin[m * 64 + c], u = fin[m * 64 + c + 32];
      const float h = g / (1.f + expf(-g)) * u;
      p.out16[(long long)(m0 + m) * p.ldo16 + fc] = f2bf(h);
    }
  }
}

const char* gv_name(int pro, int epi) {
  if (epi == EPI_QKV) return "gemv_qkv_rope_append";
  if (epi == EPI_SWIGLU) return "gemv_gateup_swiglu";
  if (epi == EPI_BF16) return "gemv_stage2";
  return pro == PRO_RMSNORM ? "gemv_stage1_rmsnorm" : "gemv_stage1";
}

// Bytes one launch must move: every factor element once, the activation
// rows once, the outputs once (a residual is read once more).
double gv_bytes(const GvParams& p, int pro, int epi) {
  double b = 0.0;
  for (int i = 0; i < p.nprob; ++i) {
    const double kn = (double)p.K * p.prob[i].N;
    b += 2.0 * kn * (epi == EPI_SWIGLU ? 2.0 : 1.0);
    b += (double)p.M * p.prob[i].N * (epi == EPI_F32 ? 4.0 : 2.0);
  }
  const double a_elems = (double)p.M * p.K * (epi == EPI_SWIGLU ? 2.0 : 1.0) *
                         (pro == PRO_F32 ? (epi == EPI_QKV ? 3.0 : 1.0) : 1.0);
  b += a_elems * (pro == PRO_F32 ? 4.0 : 2.0);
  if (p.resid) b += 2.0 * p.M * p.prob[0].N;
  return b;
}

template <int MT, int PRO, int EPI, int MAP>
int launch_one(const GvParams& p, int total_tiles, cudaStream_t stream) {
  constexpr int NSEG = (MAP == MAP_SWIGLU) ? 2 : 1;
  const size_t smem = (size_t)(NSEG * MT * p.KC + 8 * MT * 64) * sizeof(float) +
                      (size_t)p.KC * 64 * sizeof(bf16);
  auto kern = gemv_splitk_kernel<MT, PRO, EPI, MAP>;
  static SmemAttrOnce smem_once;  // per instantiation, per device
  FSVD_TRY(set_smem_once(smem_once, kern, 200 * 1024));
  if (smem > 200 * 1024) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  double flops = 0.0;
  for (int i = 0; i < p.nprob; ++i)
    flops += 2.0 * p.M * (double)p.K * p.prob[i].N * (EPI == EPI_SWIGLU ? 2.0 : 1.0);
  const LaunchTag tag{gv_name(PRO, EPI), gv_bytes(p, PRO, EPI), flops};
  return launch_pdl(tag, kern, dim3(total_tiles, p.splits, ceil_div(p.M, MT)), dim3(GV_THREADS), smem, stream, p);
}

template <int PRO, int EPI, int MAP>
int launch_mt(const GvParams& p, int total_tiles, cudaStream_t stream) {
  if (p.M <= 1) return launch_one<1, PRO, EPI, MAP>(p, total_tiles, stream);
  if (p.M <= 2) return launch_one<2, PRO, EPI, MAP>(p, total_tiles, stream);
  if (p.M <= 4) return launch_one<4, PRO, EPI, MAP>(p, total_tiles, stream);
  return launch_one<8, PRO, EPI, MAP>(p, total_tiles, stream);
}

}  // namespace

int gemv_tiles_for(int map, int N, int D) {
  if (map == MAP_SWIGLU) return ceil_div(N, 32);
  if (map == MAP_ROPE) return (N / D) * (D / 64);
  return ceil_div(N, 64);
}

int gemv_launch(GvParams p, int pro, int epi, int map, int total_rows,
                int target_ctas, cudaStream_t stream) {
  int tiles = 0;
  for (int i = 0; i < p.nprob; ++i) {
    p.tile_start[i] = tiles;
    tiles += gemv_tiles_for(map, p.prob[i].N, p.D);
  }
  for (int i = p.nprob; i < 4; ++i) p.tile_start[i] = tiles;
  // One launch for all rows: groups of up to 8 rows are the third grid
  // dimension (each CTA of a group re-reads its factor block, from L2 after
  // the first).  Split K so that about `target_ctas` CTAs (one resident
  // wave) cover the launch, with at most 512 factor rows (64 KB) per CTA.
  const int groups = ceil_div(total_rows, 8);
  const int slots = tiles * groups;
  int splits = target_ctas / (slots > 0 ? slots : 1);
  splits = splits < 1 ? 1 : splits;
  const int max_splits = ceil_div(p.K, 32);
  splits = splits > max_splits ? max_splits : splits;
  p.KC = round_up(ceil_div(p.K, splits), 32);
  p.KC = p.KC > 512 ? 512 : p.KC;
  p.splits = ceil_div(p.K, p.KC);
  const int mt = total_rows <= 1 ? 1 : (total_rows <= 2 ? 2 : (total_rows <= 4 ? 4 : 8));
  if ((long long)slots > p.counters_cap ||
      (p.splits > 1 && (long long)slots * p.splits * (mt * 64 + 8) > p.part_cap))
    return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  {
    p.m0 = 0;
    p.M = total_rows;
    int st = FLASHSVD_ERR_INVALID_ARG;
#define FSVD_GV(PRO_, EPI_, MAP_) \
    if (pro == PRO_ && epi == EPI_ && map == MAP_) st = launch_mt<PRO_, EPI_, MAP_>(p, tiles, stream);
    FSVD_GV(PRO_RMSNORM, EPI_F32, MAP_PLAIN)
    FSVD_GV(PRO_BF16, EPI_F32, MAP_PLAIN)
    FSVD_GV(PRO_F32, EPI_BF16, MAP_PLAIN)
    FSVD_GV(PRO_F32, EPI_QKV, MAP_ROPE)
    FSVD_GV(PRO_F32, EPI_SWIGLU, MAP_SWIGLU)
#undef FSVD_GV
    if (st != FLASHSVD_OK) return st;
  }
  return FLASHSVD_OK;
}

}  // namespace fsvd
