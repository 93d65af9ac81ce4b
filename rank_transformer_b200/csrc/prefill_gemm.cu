// Prefill-regime (M > 32) factorized linear on the 5th-generation tensor
// cores.
//
// FlashSVD v1.5 (gist.science explainer), Technical Summary, Problem
// Statement: prefill is arithmetic-bound and benefits from the reduced FLOPs
// of y = (x U) V, so both stages are dense tensor-core contractions.
//
// tc_gemm_kernel: persistent, warp-specialised C = A . B, A [M x K] bf16
// K-major, B [K x N] bf16 MN-major (row-major factors as stored), fp32
// accumulation in tensor memory.
//   warp 0      one thread issues TMA loads of A [128 x 64] and B [64 x BN]
//               tiles (128-byte swizzle) into a STAGES-deep ring;
//   warp 1      allocates tensor memory; one thread issues tcgen05.mma
//               (M=128, N=BN, K=16) into one of two accumulator buffers and
//               frees ring slots / publishes finished tiles with
//               tcgen05.commit;
//   warps 2..9  read the accumulator with tcgen05.ld (two warps per TMEM
//               lane quadrant, alternate 64-column pairs), apply the fused
//               epilogue and store.
// A grouped launch runs up to three GEMMs that share A (q, k, v stage 1):
// their column tiles follow one another, each with its own B and output.
// Every wait is bounded: on expiry the CTA raises the device status word
// and winds down (waits for its own copies, frees tensor memory).
#include <cstring>

#include "kernels.h"
#include "tc.cuh"

namespace fsvd {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 tensor map: [rows x cols] with row stride ld elements, box of
// box_cols x box_rows, optional 128-byte swizzle; out-of-range elements
// load as zero.
int encode_map(CUtensorMap* map, const void* base, long long rows, long long cols, long long ld,
               int box_cols, int box_rows, bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return FLASHSVD_ERR_CUDA;
  if (!aligned16(base) || (ld * 2) % 16 != 0) return FLASHSVD_ERR_MISALIGNED;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1u, 1u};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                        box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FLASHSVD_OK : FLASHSVD_ERR_INVALID_ARG;
}

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int TC_THREADS = 320;  // TMA warp, MMA warp, 8 epilogue warps

struct TcArgs {
  int M, N, K;          // per half for the dual (SwiGLU) form
  int tiles_m, tiles_n;
  int a2, b2;           // dual: A column / B row offset of the second half
  const bf16* bias;
  const bf16* resid; long long ldr;
  bf16* y; long long ldy;
  float* y32;
  int kind; bf16* cache; int S, S_max, HD, D;
  const float* rope_cos; const float* rope_sin;
  int* status;
  // Stage 2 of a factorized linear: the rank activation z (A operand, rows of
  // zld elements) is dead once every column tile of a 128-row block has
  // consumed it; the last CTA to finish a block (counter zcnt[block], zero
  // between launches) discards the block's L2 lines, so z is never written
  // back to HBM.
  const bf16* zdrop; long long zld; int* zcnt;
  // Grouped form (plain bf16 epilogue only): nprob problems share A; the
  // global column-tile index runs over problem 0's tiles, then 1's, then
  // 2's (first tile pt[i]); problem i has B map i, output gy[i] (row
  // stride gldy[i]) and width gN[i].  nprob <= 1: a.y, a.ldy, a.N.
  int nprob; int pt[3];
  bf16* gy[3]; long long gldy[3]; int gN[3];
  // Grouped q/k/v stage 2 (QKV epilogue): problem i reads A rows from
  // grow[i] (the rank activations stacked in one buffer), has epilogue kind
  // gkind[i] (0 q -> gy[i], 1 k, 2 v -> gcache[i]), bias gbias[i] and RoPE
  // when grope[i].
  int grow[3]; int gkind[3]; bf16* gcache[3]; const bf16* gbias[3]; int grope[3];
};

// Problem of global column tile gn of a grouped launch, and its first tile.
__device__ __forceinline__ int group_of(const TcArgs& a, int gn) {
  return a.nprob <= 1 ? 0 : (gn >= a.pt[1]) + (a.nprob > 2 && gn >= a.pt[2]);
}

// GELU(v) = v * Phi(v) = 0.5 v (1 + erf(v / sqrt 2)), with erf from
// Abramowitz & Stegun, Handbook of Mathematical Functions, formula 7.1.26:
// erf(x) = 1 - (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-x^2),
// t = 1 / (1 + p x), x >= 0 (odd extension), |error| <= 1.5e-7 -- below the
// bf16 rounding of the output, and branch-free (one reciprocal, one exp2);
// gelu_erf2 below evaluates it on two values with packed fp32x2 arithmetic.

// Packed fp32x2 helpers: (a0, a1) op (b0, b1) [op (c0, c1)] in one instruction.
__device__ __forceinline__ void fma_x2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                       float c1) {
  asm("{\n\t.reg .b64 aa, bb, cc;\n\t"
      "mov.b64 aa, {%2, %3};\n\t"
      "mov.b64 bb, {%4, %5};\n\t"
      "mov.b64 cc, {%6, %7};\n\t"
      "fma.rn.f32x2 aa, aa, bb, cc;\n\t"
      "mov.b64 {%0, %1}, aa;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void mul_x2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 aa, bb;\n\t"
      "mov.b64 aa, {%2, %3};\n\t"
      "mov.b64 bb, {%4, %5};\n\t"
      "mul.rn.f32x2 aa, aa, bb;\n\t"
      "mov.b64 {%0, %1}, aa;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void gelu_erf2(float& v0, float& v1) {
  float x0, x1;
  mul_x2(x0, x1, fabsf(v0), fabsf(v1), 0.70710678118654752f, 0.70710678118654752f);
  float d0, d1, t0, t1;
  fma_x2(d0, d1, 0.3275911f, 0.3275911f, x0, x1, 1.f, 1.f);
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t0) : "f"(d0));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t1) : "f"(d1));
  float p0, p1;
  fma_x2(p0, p1, 1.061405429f, 1.061405429f, t0, t1, -1.453152027f, -1.453152027f);
  fma_x2(p0, p1, p0, p1, t0, t1, 1.421413741f, 1.421413741f);
  fma_x2(p0, p1, p0, p1, t0, t1, -0.284496736f, -0.284496736f);
  fma_x2(p0, p1, p0, p1, t0, t1, 0.254829592f, 0.254829592f);
  mul_x2(p0, p1, p0, p1, t0, t1);
  float q0, q1, e0, e1;
  mul_x2(q0, q1, x0, x1, x0, x1);
  mul_x2(q0, q1, q0, q1, -1.4426950408889634f, -1.4426950408889634f);
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e0) : "f"(q0));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(q1));
  float a0, a1;  // erf(|x|)
  fma_x2(a0, a1, -p0, -p1, e0, e1, 1.f, 1.f);
  a0 = copysignf(a0, v0);
  a1 = copysignf(a1, v1);
  float h0, h1;  // 0.5 v
  mul_x2(h0, h1, v0, v1, 0.5f, 0.5f);
  fma_x2(v0, v1, h0, h1, a0, a1, h0, h1);  // 0.5 v (1 + erf) = 0.5 v + 0.5 v erf
}

__device__ __forceinline__ void store8(bf16* p, const float* v) {
  uint4 u;
  u.x = pack_bf2(v[0], v[1]); u.y = pack_bf2(v[2], v[3]);
  u.z = pack_bf2(v[4], v[5]); u.w = pack_bf2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void load8(const bf16* p, float* v) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  v[0] = bf_lo(u.x); v[1] = bf_hi(u.x); v[2] = bf_lo(u.y); v[3] = bf_hi(u.y);
  v[4] = bf_lo(u.z); v[5] = bf_hi(u.z); v[6] = bf_lo(u.w); v[7] = bf_hi(u.w);
}

// PAIR: one CTA of a 2-SM pair, which holds half of the tile's BN columns
// of B (the other CTA the other half) and its own 128 rows of A.
template <int BN, int STAGES, bool DUAL, bool PAIR = false>
struct Layout {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BK * (PAIR ? BN / 2 : BN) * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  static constexpr int SMEM = 1024 + BAR_OFF + 256;  // + alignment slack
  static constexpr int ACC_COLS = DUAL ? 2 * BN : BN;
  // accumulator buffers: two (the epilogue of a tile overlaps the next
  // tile's main loop) unless one accumulator fills the 512 columns
  static constexpr int NBUF = 2 * ACC_COLS <= 512 ? 2 : 1;
  static constexpr int TMEM_COLS = NBUF * ACC_COLS;
  // allocations are powers of 2 of at least 32 columns
  static constexpr int TMEM_ALLOC = TMEM_COLS <= 256 ? 256 : 512;
  static_assert(TMEM_COLS <= 512, "tensor memory: 512 columns");
};

// PAIR: launched in clusters of 2; each pair computes a 256 x BN tile with
// the 2-SM MMA (cta_group::2): the leader (rank 0) issues it and owns the
// operand-full barriers, both CTAs load their halves of A and B (for the
// dual form, half of the gate columns and half of the up columns) and run
// the epilogue of their 128 rows.  Tiles are counted per pair (a.tiles_m =
// ceil(M / 256)).
template <int BN, int STAGES, bool DUAL, int EPI, bool PAIR = false>
__global__ void __launch_bounds__(TC_THREADS, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmB2,
               const __grid_constant__ TcArgs a) {
  using L = Layout<BN, STAGES, DUAL, PAIR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = a.tiles_m * a.tiles_n;
  const int nkb = (a.K + BK - 1) / BK;
  const int kb_total = DUAL ? 2 * nkb : nkb;
  constexpr uint32_t IDESC = tc::idesc_bf16(BN, true, PAIR ? 256 : 128);
  // pair: rank in the pair, the pair's index and count
  const uint32_t rank = PAIR ? tc::cluster_ctarank() : 0u;
  const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  constexpr int TM = PAIR ? 2 * BM : BM;   // rows per tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(full + s, 1);
      tc::mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(tfull + b, 1);
      tc::mbar_init(tempty + b, PAIR ? 16 : 8);   // the epilogue warps of both CTAs
    }
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tmA);
    tc::tma_prefetch_desc(&tmB);
    if (a.nprob > 1) tc::tma_prefetch_desc(&tmB1);
    if (a.nprob > 2) tc::tma_prefetch_desc(&tmB2);
  }
  if (warp == 1) {
    if (PAIR) {
      tc::tmem_alloc_pair(tmem_holder, L::TMEM_ALLOC);
      tc::tmem_relinquish_pair();
    } else {
      tc::tmem_alloc(tmem_holder, L::TMEM_ALLOC);
      tc::tmem_relinquish();
    }
    tc::fence_before_sync();
  }
  __syncthreads();
  // pair: the peer's loads signal the leader's barriers and the leader's
  // MMAs write the peer's tensor memory: both must be set up first
  if (PAIR) tc::cluster_sync();
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;

  pdl_launch_dependents();
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = unit; t < tiles && ok; t += units) {
        const int gn = t / a.tiles_m, gp = group_of(a, gn);
        const int m0 = (t % a.tiles_m) * TM + (int)rank * BM, n0 = (gn - (gp ? a.pt[gp] : 0)) * BN;
        const CUtensorMap* mB = gp == 0 ? &tmB : (gp == 1 ? &tmB1 : &tmB2);
        for (int kb = 0; kb < kb_total; ++kb) {
          if (!tc::mbar_wait(empty + stage, phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
          const bool second = DUAL && kb >= nkb;
          const int kk = second ? kb - nkb : kb;
          const int ka = (second ? a.a2 : 0) + kk * BK;
          const int kr = (second ? a.b2 : 0) + kk * BK;
          uint8_t* sA = smem + stage * L::STAGE_BYTES;
          uint8_t* sB = sA + L::A_BYTES;
          const int arow = m0 + (a.nprob > 1 ? a.grow[gp] : 0);
          if (PAIR) {
            // both halves complete on the leader's barrier, which expects
            // the bytes of both CTAs
            const uint32_t fb = tc::mapa_shared(tc::smem_u32(full + stage), 0);
            if (rank == 0) tc::mbar_expect_tx(full + stage, 2 * L::STAGE_BYTES);
            tc::tma_load_2d_pair(sA, &tmA, fb, ka, arow);
#pragma unroll
            for (int j = 0; j < BN / 128; ++j)
              tc::tma_load_2d_pair(sB + j * 8192, mB, fb, n0 + (int)rank * (BN / 2) + 64 * j, kr);
          } else {
            tc::mbar_expect_tx(full + stage, L::STAGE_BYTES);
            tc::tma_load_2d(sA, &tmA, full + stage, ka, arow);
#pragma unroll
            for (int j = 0; j < BN / 64; ++j) tc::tma_load_2d(sB + j * 8192, mB, full + stage, n0 + 64 * j, kr);
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok && rank == 0) {
        // Winding down: let this CTA's copies that are still in flight land
        // before shared memory is released (bounded, ignores the flag).  A
        // pair's copies all complete on the leader's barriers; the peer is
        // held by the final cluster barrier instead.
        const int outstanding = issued < STAGES ? issued : STAGES;
        for (int i = 1; i <= outstanding; ++i) {
          int s = stage - i;
          uint32_t ph = phase;
          if (s < 0) { s += STAGES; ph ^= 1u; }
          const long long t0 = clock64();
          while (!tc::mbar_try_wait(full + s, ph) && clock64() - t0 < tc::kWaitCycles) {}
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = unit; t < tiles && ok; t += units, ++it) {
        const int buf = it % L::NBUF;
        const uint32_t tph = (uint32_t)(it / L::NBUF) & 1u;
        if (!tc::mbar_wait(tempty + buf, tph ^ 1u, abort_flag, a.status)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t d0 = tmem_base + (uint32_t)(buf * L::ACC_COLS);
        for (int kb = 0; kb < kb_total; ++kb) {
          if (!tc::mbar_wait(full + stage, phase, abort_flag, a.status)) { ok = false; break; }
          tc::fence_after_sync();
          const bool second = DUAL && kb >= nkb;
          const uint32_t d = second ? d0 + BN : d0;
          const bool first = (kb == 0) || (DUAL && kb == nkb);
          const uint32_t sa = tc::smem_u32(smem + stage * L::STAGE_BYTES);
          const uint32_t sb = sa + L::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = tc::sdesc_sw128(sa + k * 32, 16, 1024);
            const uint64_t bd = tc::sdesc_sw128(sb + k * 2048, 8192, 1024);
            if (PAIR)
              tc::mma_bf16_pair(d, ad, bd, IDESC, (first && k == 0) ? 0u : 1u);
            else
              tc::mma_bf16(d, ad, bd, IDESC, (first && k == 0) ? 0u : 1u);
          }
          // the stage is free in both CTAs of a pair
          if (PAIR)
            tc::mma_commit_pair_mc(empty + stage, (uint16_t)3);
          else
            tc::mma_commit(empty + stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (ok) {
          if (PAIR)
            tc::mma_commit_pair_mc(tfull + buf, (uint16_t)3);
          else
            tc::mma_commit(tfull + buf);
        }
      }
      // Every MMA this thread issued has completed once `drain` fires.
      if (PAIR)
        tc::mma_commit_pair(drain);
      else
        tc::mma_commit(drain);
      const long long t0 = clock64();
      while (!tc::mbar_try_wait(drain, 0) && clock64() - t0 < tc::kWaitCycles) {}
    }
  } else {
    // --------------------------------------------------------- epilogue --
    // Warp w reads TMEM lanes 32 (w % 4) .. + 31 (its 32 rows); the two
    // warps of a lane quadrant take alternate 32-column chunks of the tile.
    const int q = warp & 3;
    const int part = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    int it = 0;
    for (int t = unit; t < tiles; t += units, ++it) {
      const int buf = it % L::NBUF;
      const uint32_t tph = (uint32_t)(it / L::NBUF) & 1u;
      if (!tc::mbar_wait(tfull + buf, tph, abort_flag, a.status)) break;
      tc::fence_after_sync();
      const int gn = t / a.tiles_m, gp = group_of(a, gn);
      const int m0 = (t % a.tiles_m) * TM + (int)rank * BM, n0 = (gn - (gp ? a.pt[gp] : 0)) * BN;
      // this tile's output (grouped launches: its problem's)
      bf16* const ty = a.nprob > 1 ? a.gy[gp] : a.y;
      const long long tldy = a.nprob > 1 ? a.gldy[gp] : a.ldy;
      const int tN = a.nprob > 1 ? a.gN[gp] : a.N;
      const int m = m0 + row;
      const bool mok = m < a.M;
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * L::ACC_COLS);

      if (EPI == PF_EPI_QKV) {
        // RoPE pairs columns i and i + D/2 of a head: process a first-half
        // chunk of 32 columns together with its partner chunk.
        const int half = a.D >> 1;
        const int hc = half >> 5;  // chunks per half head
        const int bq = mok ? m / a.S : 0, tq = mok ? m - bq * a.S : 0;
        // this tile's problem (grouped q/k/v: its kind, cache, bias, RoPE)
        const bool grp = a.nprob > 1;
        const int kind = grp ? a.gkind[gp] : a.kind;
        bf16* const cache = grp ? a.gcache[gp] : a.cache;
        const bf16* const bias = grp ? a.gbias[gp] : a.bias;
        const bool rope = grp ? (a.grope[gp] != 0) : (a.rope_cos != nullptr);
        int pair = 0;
        for (int c = 0; c < BN / 32; ++c) {
          if ((c % (2 * hc)) >= hc) continue;  // second-half chunks ride along
          if ((pair++ & 1) != part) continue;
          const int n = n0 + c * 32;
          uint32_t r0[32], r1[32];
          tc::tmem_ld32(tb + c * 32, r0);
          tc::tmem_ld32(tb + (c + hc) * 32, r1);
          tc::tmem_ld_wait();
          if (!mok || n >= a.N) continue;
          float lo[32], hi[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) { lo[j] = __uint_as_float(r0[j]); hi[j] = __uint_as_float(r1[j]); }
          if (bias) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              float b0[8], b1[8];
              load8(bias + n + 8 * g, b0);
              load8(bias + n + half + 8 * g, b1);
#pragma unroll
              for (int j = 0; j < 8; ++j) { lo[8 * g + j] += b0[j]; hi[8 * g + j] += b1[j]; }
            }
          }
          if (rope) {
            // 32 consecutive angles of this row's position: 16-byte loads.
            const int i0 = n % a.D;
            const float4* cs = reinterpret_cast<const float4*>(a.rope_cos + (long long)tq * half + i0);
            const float4* sn = reinterpret_cast<const float4*>(a.rope_sin + (long long)tq * half + i0);
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              const float4 c4 = __ldg(cs + j4), s4 = __ldg(sn + j4);
              const float cj[4] = {c4.x, c4.y, c4.z, c4.w}, sj[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int j = 4 * j4 + e;
                const float l2 = lo[j] * cj[e] - hi[j] * sj[e];
                hi[j] = hi[j] * cj[e] + lo[j] * sj[e];
                lo[j] = l2;
              }
            }
          }
          bf16* dst = kind == 0 ? ty + (long long)m * tldy
                                : cache + ((long long)bq * a.S_max + tq) * a.HD;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            store8(dst + n + 8 * g, lo + 8 * g);
            store8(dst + n + half + 8 * g, hi + 8 * g);
          }
        }
      } else {
        // A warp owns pairs of chunks (64 columns: whole 128-byte lines of
        // a row), so no output line is shared between the two warps of a
        // quadrant.  Residual and bias are read before the accumulator
        // wait: the residual may be the output buffer itself (in-place
        // update), and reading it up front keeps the loads off the stores.
        for (int c = 0; c < BN / 32; ++c) {
          if (((c >> 1) & 1) != part) continue;
          const int n = n0 + c * 32;
          constexpr bool PLAIN = !DUAL && EPI != PF_EPI_F32;
          uint4 rr[PLAIN ? 4 : 1], bb[PLAIN ? 4 : 1];
          if (PLAIN) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const int ng = n + 8 * g;
              const bool in = mok && ng < tN;
              rr[g] = (in && a.resid) ? *reinterpret_cast<const uint4*>(a.resid + (long long)m * a.ldr + ng)
                                      : make_uint4(0u, 0u, 0u, 0u);
              bb[g] = (in && a.bias) ? *reinterpret_cast<const uint4*>(a.bias + ng) : make_uint4(0u, 0u, 0u, 0u);
            }
          }
          __syncwarp();
          uint32_t r0[32];
          uint32_t r1[DUAL ? 32 : 1];
          tc::tmem_ld32(tb + c * 32, r0);
          if (DUAL) tc::tmem_ld32(tb + BN + c * 32, r1);
          tc::tmem_ld_wait();
          if (!mok) continue;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int ng = n + 8 * g;
            if (ng >= tN) break;
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r0[8 * g + j]);
            if (EPI == PF_EPI_F32) {
              float4* dst = reinterpret_cast<float4*>(a.y32 + (long long)m * a.ldy + ng);
              dst[0] = make_float4(v[0], v[1], v[2], v[3]);
              dst[1] = make_float4(v[4], v[5], v[6], v[7]);
              continue;
            }
            if (DUAL) {
              // SiLU(g) * u = g u / (1 + 2^(-g log2 e)): hardware exp2
              // approximation and reciprocal (relative error ~2^-22, far
              // below the bf16 rounding of the output)
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float u = __uint_as_float(r1[8 * g + j]);
                float e, rc;
                asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(v[j] * -1.4426950408889634f));
                asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rc) : "f"(1.f + e));
                v[j] = v[j] * rc * u;
              }
            } else {
              const int gi = PLAIN ? g : 0;
              const uint32_t bw[4] = {bb[gi].x, bb[gi].y, bb[gi].z, bb[gi].w};
              const uint32_t rw[4] = {rr[gi].x, rr[gi].y, rr[gi].z, rr[gi].w};
              if (a.bias) {
#pragma unroll
                for (int j = 0; j < 4; ++j) { v[2 * j] += bf_lo(bw[j]); v[2 * j + 1] += bf_hi(bw[j]); }
              }
              if (EPI == PF_EPI_GELU) {
#pragma unroll
                for (int j = 0; j < 8; j += 2) gelu_erf2(v[j], v[j + 1]);
              }
              if (a.resid) {
#pragma unroll
                for (int j = 0; j < 4; ++j) { v[2 * j] += bf_lo(rw[j]); v[2 * j + 1] += bf_hi(rw[j]); }
              }
            }
            store8(ty + (long long)m * tldy + ng, v);
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if (PAIR)   // the accumulator buffer spans both CTAs: release it at the leader
          tc::mbar_arrive_cluster(tc::mapa_shared(tc::smem_u32(tempty + buf), 0));
        else
          tc::mbar_arrive(tempty + buf);
      }
      if (a.zdrop && q == 0 && part == 0) {
        // This tile's MMAs are complete: every TMA read of its z rows is
        // done.  One warp counts the block's finished column tiles; the last
        // CTA's warp discards the block's z lines (whole 128-byte lines
        // inside rows [m0, m0 + 128) only).
        // (grouped: counters and rows per problem, whose A rows start at
        // grow[gp] and whose column tiles are pt[gp] .. pt[gp + 1])
        const int gtn = a.nprob > 1 ? (gp + 1 < a.nprob ? a.pt[gp + 1] : a.tiles_n) - a.pt[gp] : a.tiles_n;
        const int mb = (a.nprob > 1 ? gp * a.tiles_m * (TM / BM) : 0) + m0 / BM;
        const long long zr = a.nprob > 1 ? a.grow[gp] : 0;
        const unsigned act = __activemask();
        int last = 0;
        if (lane == 0) {
          last = atomicAdd(a.zcnt + mb, 1) == gtn - 1;
          if (last) a.zcnt[mb] = 0;
        }
        last = __shfl_sync(act, last, __ffs(act) - 1);
        if (last) {
          const long long b0 = (zr + m0) * a.zld * 2;
          const long long b1 = (zr + min(m0 + BM, a.M)) * a.zld * 2;
          const uintptr_t base = reinterpret_cast<uintptr_t>(a.zdrop);
          const uintptr_t l0 = (base + b0 + 127) & ~(uintptr_t)127, l1 = (base + b1) & ~(uintptr_t)127;
          for (uintptr_t ln = l0 + (uintptr_t)lane * 128; ln < l1; ln += 32 * 128)
            asm volatile("discard.global.L2 [%0], 128;" ::"l"(ln) : "memory");
        }
      }
    }
  }

  __syncthreads();
  // pair: the leader's MMAs have drained and both epilogues have read their
  // tensor memory before either CTA frees it
  if (PAIR) tc::cluster_sync();
  if (warp == 1) {
    tc::fence_after_sync();
    if (PAIR)
      tc::tmem_dealloc_pair(tmem_base, L::TMEM_ALLOC);
    else
      tc::tmem_dealloc(tmem_base, L::TMEM_ALLOC);
  }
}

// ------------------------------------------------------------- host ----

// bf16 matrix [rows x cols], row stride ld elements; box = 64 columns x box_rows rows.
int make_map(CUtensorMap* map, const void* base, long long rows, long long cols, long long ld,
             int box_rows) {
  return encode_map(map, base, rows, cols, ld, 64, box_rows, true);
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

double gemm_bytes(const TcArgs& a, bool dual) {
  const double halves = dual ? 2.0 : 1.0;
  return 2.0 * ((double)a.M * a.K * halves + (double)a.K * a.N * halves + (double)a.M * a.N);
}

template <int BN, int STAGES, bool DUAL, int EPI, bool PAIR = false>
int launch_tc(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mb1, const CUtensorMap& mb2,
              TcArgs a, const char* name, cudaStream_t stream) {
  using L = Layout<BN, STAGES, DUAL, PAIR>;
  auto kern = tc_gemm_kernel<BN, STAGES, DUAL, EPI, PAIR>;
  static SmemAttrOnce smem_once;
  FSVD_TRY(set_smem_once(smem_once, kern, L::SMEM));
  a.tiles_m = ceil_div(a.M, PAIR ? 2 * BM : BM);
  if (a.nprob > 1) {
    // grouped: problem i's column tiles start at pt[i]; a.N = total width
    int nt = 0;
    a.N = 0;
    for (int i = 0; i < a.nprob; ++i) {
      a.pt[i] = nt;
      nt += ceil_div(a.gN[i], BN);
      a.N += a.gN[i];
    }
    a.tiles_n = nt;
  } else {
    a.tiles_n = ceil_div(a.N, BN);
  }
  const int tiles = a.tiles_m * a.tiles_n;
  const double flops = 2.0 * a.M * (double)a.N * a.K * (DUAL ? 2.0 : 1.0);
  const LaunchTag tag{name, gemm_bytes(a, DUAL), flops};
  if (PAIR) {
    const int pairs = sm_count() / 2;
    const int grid = 2 * (tiles < pairs ? tiles : pairs);
    return launch_pdl_cluster(tag, 2, kern, dim3(grid), dim3(TC_THREADS), (size_t)L::SMEM, stream, ma, mb, mb1,
                              mb2, a);
  }
  const int grid = tiles < sm_count() ? tiles : sm_count();
  return launch_pdl(tag, kern, dim3(grid), dim3(TC_THREADS), (size_t)L::SMEM, stream, ma, mb, mb1, mb2, a);
}

// Whether BN = 256 GEMMs of at least 256 rows run as 2-SM CTA pairs
// (cta_group::2: each CTA loads half of B, so the operand traffic into an
// SM per FLOP drops by a third).
constexpr bool kGemmPairs = true;

template <int EPI>
int launch_wide(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mb1, const CUtensorMap& mb2,
                const TcArgs& a, const char* name, cudaStream_t stream) {
  // Widths that 192-column tiles cover with less padding than 256-column
  // ones (rank-192 projections: a quarter of a 256-wide tile is empty) run
  // 192-wide single-CTA tiles (a 2-SM pair would split them into 96-column
  // halves, below the 64-column TMA box granularity).  Not for the q/k/v
  // epilogue, whose RoPE pairs columns within a head that a 192-column tile
  // may split.
  if constexpr (EPI != PF_EPI_QKV) {
    bool narrow = true;
    const int np = a.nprob > 1 ? a.nprob : 1;
    for (int i = 0; i < np; ++i) {
      const int n = a.nprob > 1 ? a.gN[i] : a.N;
      if (ceil_div(n, 192) * 192 >= ceil_div(n, 256) * 256) narrow = false;
    }
    if (narrow) return launch_tc<192, 5, false, EPI>(ma, mb, mb1, mb2, a, name, stream);
  }
  if (kGemmPairs && a.M >= 2 * BM) return launch_tc<256, 6, false, EPI, true>(ma, mb, mb1, mb2, a, name, stream);
  return launch_tc<256, 4, false, EPI>(ma, mb, mb1, mb2, a, name, stream);
}

// One tensor-core GEMM C = A . B with the given epilogue.
int gemm(const bf16* A, long long lda, long long a_cols, const bf16* B, long long ldb, long long b_rows,
         TcArgs a, int epi, bool dual, const char* name, cudaStream_t stream) {
  CUtensorMap ma, mb;
  FSVD_TRY(make_map(&ma, A, a.M, a_cols, lda, BM));
  if (dual) {
    FSVD_TRY(make_map(&mb, B, b_rows, a.N, ldb, BK));
    // 256-wide gate and up accumulators fill the 512 TMEM columns, so the
    // accumulator is single-buffered (the epilogue does not overlap the
    // next tile's main loop); 128-wide tiles with a double-buffered
    // accumulator ran their MMAs at about 57 % of the tensor-core rate and
    // took 6.1 ms per 7B prefill against 4.5 (single CTAs) and 4.2 ms
    // (2-SM pairs) for 256-wide ones.  With a short K (r_f < 1024: 2 x 16
    // k-blocks or fewer per tile) the exposed epilogue outweighs that and
    // the double-buffered 128-wide tiles stay ahead.
    if (a.K >= 1024) {
      if (kGemmPairs && a.M >= 2 * BM)
        return launch_tc<256, 6, true, PF_EPI_SWIGLU, true>(ma, mb, mb, mb, a, name, stream);
      return launch_tc<256, 4, true, PF_EPI_SWIGLU>(ma, mb, mb, mb, a, name, stream);
    }
    return launch_tc<128, 6, true, PF_EPI_SWIGLU>(ma, mb, mb, mb, a, name, stream);
  }
  FSVD_TRY(make_map(&mb, B, b_rows, a.N, ldb, BK));
  switch (epi) {
    case PF_EPI_BF16: return launch_wide<PF_EPI_BF16>(ma, mb, mb, mb, a, name, stream);
    case PF_EPI_GELU: return launch_wide<PF_EPI_GELU>(ma, mb, mb, mb, a, name, stream);
    case PF_EPI_QKV: return launch_wide<PF_EPI_QKV>(ma, mb, mb, mb, a, name, stream);
    case PF_EPI_F32: return launch_wide<PF_EPI_F32>(ma, mb, mb, mb, a, name, stream);
    default: return FLASHSVD_ERR_INVALID_ARG;
  }
}

}  // namespace

int prefill_stage1_grouped(const bf16* x, long long ldx, int d, int M, int n, const bf16* const* U,
                           const int* r, bf16* const* z, int* status, cudaStream_t stream) {
  if (n < 1 || n > 3) return FLASHSVD_ERR_INVALID_ARG;
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.M = M; a.K = d;
  a.status = status;
  a.nprob = n;
  CUtensorMap ma, mb[3];
  FSVD_TRY(make_map(&ma, x, M, d, ldx, BM));
  for (int i = 0; i < n; ++i) {
    FSVD_TRY(make_map(&mb[i], U[i], d, r[i], r[i], BK));
    a.gy[i] = z[i]; a.gldy[i] = r[i]; a.gN[i] = r[i];
  }
  a.y = z[0]; a.ldy = r[0];
  return launch_wide<PF_EPI_BF16>(ma, mb[0], mb[n > 1 ? 1 : 0], mb[n > 2 ? 2 : 0], a,
                                               "tc_stage1_xu_grouped", stream);
}

int prefill_stage1(const bf16* x, long long ldx, int d, int M, const bf16* U, int r, bf16* z, int* status,
                   cudaStream_t stream) {
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.M = M; a.N = r; a.K = d;
  a.y = z; a.ldy = r;
  a.status = status;
  return gemm(x, ldx, d, U, r, d, a, PF_EPI_BF16, false, "tc_stage1_xu", stream);
}

int prefill_qkv_stage2_grouped(const QkvGroup& g, cudaStream_t stream) {
  if (g.n < 1 || g.n > 3) return FLASHSVD_ERR_INVALID_ARG;
  if (g.D % 64 != 0 || 256 % g.D != 0) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.M = g.M; a.K = g.r;
  a.status = g.status;
  a.nprob = g.n;
  a.S = g.S; a.S_max = g.S_max; a.HD = g.HD; a.D = g.D;
  a.rope_cos = g.rope_cos; a.rope_sin = g.rope_sin;
  int rows = 0;
  CUtensorMap mb[3];
  for (int i = 0; i < g.n; ++i) {
    FSVD_TRY(make_map(&mb[i], g.V[i], g.r, g.HD, g.HD, BK));
    a.gN[i] = g.HD; a.gy[i] = g.q; a.gldy[i] = g.ldq;
    a.grow[i] = g.row[i]; a.gkind[i] = g.kind[i]; a.gcache[i] = g.cache[i]; a.gbias[i] = g.bias[i];
    a.grope[i] = (g.kind[i] < 2 && g.rope_cos) ? 1 : 0;
    rows = max(rows, g.row[i] + g.M);
  }
  CUtensorMap ma;
  FSVD_TRY(make_map(&ma, g.z, rows, g.r, g.r, BM));
  if (g.zcnt) { a.zdrop = g.z; a.zld = g.r; a.zcnt = g.zcnt; }
  return launch_wide<PF_EPI_QKV>(ma, mb[0], mb[g.n > 1 ? 1 : 0], mb[g.n > 2 ? 2 : 0], a,
                                              "tc_stage2_qkv_grouped", stream);
}

int prefill_linear_launch(const PfLinear& p, cudaStream_t stream) {
  if (!p.z) return FLASHSVD_ERR_NOT_INITIALIZED;
  const bool dual = p.epi == PF_EPI_SWIGLU;
  if (dual && (p.r % 128) != 0) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;  // r = 2 r_f, r_f % 64 == 0
  if (p.epi == PF_EPI_QKV && (p.D % 64 != 0 || 256 % p.D != 0)) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  // Stage 1: z = x . U  [M x r], rounded to bf16.
  TcArgs a1;
  memset(&a1, 0, sizeof(a1));
  a1.M = p.M; a1.N = p.r; a1.K = p.d;
  a1.y = p.z; a1.ldy = p.r;
  a1.status = p.status;
  if (!p.z_ready) FSVD_TRY(gemm(p.x, p.ldx, p.d, p.U, p.r, p.d, a1, PF_EPI_BF16, false, "tc_stage1_xu", stream));
  // Stage 2: y = epilogue(z . V).
  TcArgs a2;
  memset(&a2, 0, sizeof(a2));
  a2.M = p.M; a2.N = p.n; a2.K = dual ? p.r / 2 : p.r;
  a2.a2 = p.r / 2; a2.b2 = p.r / 2;
  a2.bias = p.bias; a2.resid = p.resid; a2.ldr = p.ldr;
  a2.y = p.y; a2.ldy = p.ldy; a2.y32 = p.y32;
  a2.kind = p.kind; a2.cache = p.cache; a2.S = p.S; a2.S_max = p.S_max; a2.HD = p.HD; a2.D = p.D;
  a2.rope_cos = p.rope_cos; a2.rope_sin = p.rope_sin;
  a2.status = p.status;
  if (p.zcnt) { a2.zdrop = p.z; a2.zld = p.r; a2.zcnt = p.zcnt; }
  const char* name = dual                  ? "tc_stage2_swiglu"
                     : p.epi == PF_EPI_QKV ? "tc_stage2_qkv_rope"
                     : p.resid             ? "tc_stage2_zv_resid"
                                           : "tc_stage2_zv";
  return gemm(p.z, p.r, p.r, p.V, p.n, p.r, a2, p.epi, dual, name, stream);
}

int prefill_dense_launch(const PfLinear& p, cudaStream_t stream) {
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.M = p.M; a.N = p.n; a.K = p.d;
  a.y32 = p.y32; a.ldy = p.ldy;
  a.status = p.status;
  return gemm(p.x, p.ldx, p.d, p.V, p.n, p.d, a, PF_EPI_F32, false, "tc_dense_f32", stream);
}

}  // namespace fsvd
