// Prefill attention on the 5th-generation tensor cores.
//
// FlashSVD v1.5 (gist.science explainer), Technical Summary, Methodology 2:
// prefill keeps its own attention kernel (the dense-KV path is the decode
// one); here it reads the same dense [B, S_max, H, D] cache the prefill's
// q/k/v epilogue wrote.  Causal (decoder) or bidirectional (encoder).
//
// Persistent CTAs (one per SM) walk the (128-query tile, batch row, head)
// items, heaviest first; 10 warps:
//   warp 0  TMA: Q once, then 128-key K and V tiles into two rings of their
//           own (K one tile ahead of V), so a K tile waits only for the S
//           MMA that read its slot and a V tile for the P V MMA;
//   warp 1  TMEM owner and MMA issuer: S = Q K^T into one of two 128-column
//           TMEM buffers, then O += P V into a D-column TMEM accumulator,
//           with P read from TMEM (the A operand of a TMEM-A MMA);
//   warps 2-9  two threads per query row (each half of the keys and of O):
//           load the row of S from TMEM (both halves, so each thread has
//           the row max without an exchange), mask, online softmax (exp2
//           domain), rescale O in TMEM when the row's reference max moves,
//           write P (bf16 pairs) into one of two 64-column TMEM buffers; at
//           the end O / l.
// S of tile j+1 and P V of tile j-1 run on the tensor cores while the
// softmax of tile j runs: the softmax waits for P V only when it rescales O
// or reuses a P buffer.  Every wait is bounded.
//
// Factorized form (QF, FlashSVD v1.5 explainer, Methodology 2, "Prefill":
// a dedicated factorized attention kernel avoids dense materialisation):
// the query tile is formed inside the kernel from the rank activation,
// Q = z_q V_q[:, head], so dense q is never written or read.  Per item the
// TMA warp streams z_q and V_q k-blocks through the K/V ring, the MMA warp
// accumulates Q in TMEM columns 384.., and the softmax warps apply RoPE
// while moving Q (bf16) into the swizzled A operand of S = Q K^T.  The last
// of the H items that read a query tile's z_q rows discards them from L2.
#include <cstring>

#include "kernels.h"
#include "tc.cuh"

namespace fsvd {
namespace {

constexpr int AT_BM = 128;   // queries per CTA
constexpr int AT_BN = 128;   // keys per tile
constexpr int AT_THREADS = 320;  // TMA warp, MMA warp, 8 softmax warps

// 2^x with the hardware approximation (relative error ~2^-22; 2^-inf = +0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// (x0, x1) -> (2^x0, 2^x1) on the FMA and integer pipes, leaving the
// special-function unit (16 results per clock per SM, the softmax's limit)
// to the other elements.  Range reduction x = j + f with j = round(x) (adding
// 1.5 * 2^23 leaves j in the low mantissa bits) and f in [-1/2, 1/2]; 2^f by
// a cubic fitted to it on that interval (relative error below 7.5e-5, well
// under the bf16 rounding of P); 2^j by adding j to the exponent field.
// Inputs are clamped at -125, so the result stays a normal number: a masked
// key (-inf) gives 2^-125 instead of 0, below every fp32 rounding step of l
// and of O.
__device__ __forceinline__ void ex2_poly2(float& x0, float& x1) {
  constexpr float C0 = 0.99992806f, C1 = 0.69326097f, C2 = 0.24261113f, C3 = 0.05517165f;
  x0 = fmaxf(x0, -125.f);
  x1 = fmaxf(x1, -125.f);
  uint32_t t0, t1;
  asm("{\n\t.reg .b64 xx, tt, jj, ff, pp, cc;\n\t"
      "mov.b64 xx, {%2, %3};\n\t"
      "mov.b64 cc, {%4, %4};\n\t"
      "add.rn.f32x2 tt, xx, cc;\n\t"           // t = x + 1.5 * 2^23
      "mov.b64 cc, {%5, %5};\n\t"
      "add.rn.f32x2 jj, tt, cc;\n\t"           // j = t - 1.5 * 2^23 (exact)
      "mov.b64 cc, {%6, %6};\n\t"
      "fma.rn.f32x2 ff, jj, cc, xx;\n\t"       // f = x - j (exact)
      "mov.b64 pp, {%7, %7};\n\t"
      "mov.b64 cc, {%8, %8};\n\t"
      "fma.rn.f32x2 pp, pp, ff, cc;\n\t"
      "mov.b64 cc, {%9, %9};\n\t"
      "fma.rn.f32x2 pp, pp, ff, cc;\n\t"
      "mov.b64 cc, {%10, %10};\n\t"
      "fma.rn.f32x2 pp, pp, ff, cc;\n\t"
      "mov.b64 {%0, %1}, pp;\n\t"
      "mov.b64 {%2, %3}, tt;\n\t}"
      : "=r"(t0), "=r"(t1), "+f"(x0), "+f"(x1)
      : "f"(12582912.f), "f"(-12582912.f), "f"(-1.f), "f"(C3), "f"(C2), "f"(C1), "f"(C0));
  // t0, t1: 2^f bits; x0, x1: the bits of t, whose low 9 bits are j
  x0 = __uint_as_float(t0 + (__float_as_uint(x0) << 23));
  x1 = __uint_as_float(t1 + (__float_as_uint(x1) << 23));
}
// Of every 4 element pairs of a row's P, this many take ex2_poly2.
constexpr int AT_EMU = 1;

// max(a, b, c) in one instruction.
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// (a0, a1) += (b0, b1) as one packed fp32x2 add.
__device__ __forceinline__ void add2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 aa, bb;\n\t"
      "mov.b64 aa, {%0, %1};\n\t"
      "mov.b64 bb, {%2, %3};\n\t"
      "add.rn.f32x2 aa, aa, bb;\n\t"
      "mov.b64 {%0, %1}, aa;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}
// (x0, x1) * s + (c, c) as one packed fp32x2 FMA.
__device__ __forceinline__ void fma2_sc(float& x0, float& x1, float sc, float c) {
  asm("{\n\t.reg .b64 xx, ss, cc;\n\t"
      "mov.b64 xx, {%0, %1};\n\t"
      "mov.b64 ss, {%2, %2};\n\t"
      "mov.b64 cc, {%3, %3};\n\t"
      "fma.rn.f32x2 xx, xx, ss, cc;\n\t"
      "mov.b64 {%0, %1}, xx;\n\t}"
      : "+f"(x0), "+f"(x1)
      : "f"(sc), "f"(c));
}

template <int D>
struct AtLayout {
  static constexpr int KB = D / 64;              // 64-column blocks of a head
  static constexpr int TILE = AT_BN * 128;       // one [128 x 64] bf16 block, 16 KB
  static constexpr int NST = D == 64 ? 4 : 3;    // stages of the K ring and of the V ring
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + KB * TILE;
  static constexpr int V_OFF = K_OFF + NST * KB * TILE;
  static constexpr int BAR_OFF = V_OFF + NST * KB * TILE;
  static constexpr int X_OFF = BAR_OFF + 512;     // [2 halves][128] row sums l
  static constexpr int SMEM = 1024 + X_OFF + 2 * 128 * 4;
  static_assert(SMEM <= 232448, "shared memory budget");
};
// TMEM columns: S buffers [0, 128) and [128, 256), O [256, 256 + D), P
// buffers (bf16 pairs, 64 columns each) [384, 448) and [448, 512); the
// factorized form accumulates Q in [384, 384 + D), over the P buffers,
// between the previous item's last P V and the item's first P.
constexpr uint32_t AT_TM_O = 256;
constexpr uint32_t AT_TM_P = 384;

struct AtParams {
  int B, S, H, S_max;
  float scale_log2;
  bf16* out;      // [B*S x H*D]
  int* status;
  // factorized form: z_q [B*S x r] (row stride ldz) in k-blocks of 64,
  // rotary tables [S x D/2], per (batch row, query tile) discard counters
  int nq;         // r / 64
  const bf16* zq; long long ldz;
  const float* rope_cos; const float* rope_sin;
  int* zcnt;      // null: no discard
};

template <int D, bool CAUSAL, bool QF>
__global__ void __launch_bounds__(AT_THREADS, 1)
attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmVq,
                       const __grid_constant__ AtParams p) {
  using L = AtLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  constexpr int NST = L::NST;
  uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* k_full = q_full + 1;     // [NST]
  uint64_t* k_empty = k_full + NST;  // [NST]
  uint64_t* v_full = k_empty + NST;  // [NST]
  uint64_t* v_empty = v_full + NST;  // [NST]
  uint64_t* s_full = v_empty + NST;  // [2]
  uint64_t* s_empty = s_full + 2;    // [2]
  uint64_t* p_full = s_empty + 2;    // [2] P buffer written (count 8)
  uint64_t* o_done = p_full + 2;     // [2] P V of a tile using that P buffer done
  uint64_t* drain = o_done + 2;
  uint64_t* q_empty = drain + 1;     // the item's S MMAs are done: Q may be reloaded
  uint64_t* o_free = q_empty + 1;    // the epilogue has read O (count 8)
  uint64_t* qacc_full = o_free + 1;  // QF: the item's Q = z_q V_q is in TMEM
  uint64_t* qacc_free = qacc_full + 1;  // QF: the softmax warps have read it (count 8)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(qacc_free + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Persistent: work item k = (query tile, batch row, head), heaviest
  // (longest causal) query tiles first.  CTA c of G takes one item per round
  // of G, in snake order (round i: item i G + c, or i G + G - 1 - c when i
  // is odd), which pairs heavy causal tiles with light ones: at 16 query
  // tiles x 32 heads on 148 CTAs the longest CTA walks 31 key tiles (the
  // mean is 29.4) instead of 38 with a plain stride.
  // Barrier phases run on across items: T counts this CTA's key tiles, I
  // its items.
  const int qtiles = (p.S + AT_BM - 1) / AT_BM;
  const int BH = p.B * p.H;
  const int NW = qtiles * BH;
  const int G = gridDim.x, cta = blockIdx.x;
  const int full_rounds = NW / G, rem = NW - full_rounds * G;
  const int n_items =
      full_rounds + ((rem > 0 && ((full_rounds & 1) ? (G - 1 - cta) < rem : cta < rem)) ? 1 : 0);
  auto item_k = [&](int i) { return i * G + ((i & 1) ? G - 1 - cta : cta); };
  const int nt_all = (p.S + AT_BN - 1) / AT_BN;
  struct Item { int b, h, m0, nt; };
  auto item_of = [&](int k) {
    Item it;
    const int qt = qtiles - 1 - k / BH, bh = k - (k / BH) * BH;
    it.b = bh / p.H;
    it.h = bh - it.b * p.H;
    it.m0 = qt * AT_BM;
    it.nt = CAUSAL ? min(nt_all, (it.m0 + AT_BM + AT_BN - 1) / AT_BN) : nt_all;
    return it;
  };

  // QF: k-blocks of 64 of the rank, KB of them per ring stage
  const int nqs = QF ? (p.nq + L::KB - 1) / L::KB : 0;
  if (threadIdx.x == 0) {
    tc::mbar_init(q_full, QF ? 8 : 1);
    tc::mbar_init(qacc_full, 1);
    tc::mbar_init(qacc_free, 8);
    for (int i = 0; i < NST; ++i) {
      tc::mbar_init(k_full + i, 1);
      tc::mbar_init(k_empty + i, 1);
      tc::mbar_init(v_full + i, 1);
      tc::mbar_init(v_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(s_full + i, 1);
      tc::mbar_init(s_empty + i, 8);
      tc::mbar_init(p_full + i, 8);
      tc::mbar_init(o_done + i, 1);
    }
    tc::mbar_init(drain, 1);
    tc::mbar_init(q_empty, 1);
    tc::mbar_init(o_free, 8);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tmQ);
    tc::tma_prefetch_desc(&tmK);
    tc::tma_prefetch_desc(&tmV);
    if (QF) tc::tma_prefetch_desc(&tmVq);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_holder, 512);
    tc::tmem_relinquish();
    tc::fence_before_sync();
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  pdl_launch_dependents();
  pdl_wait();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA --
    if (lane == 0) {
      // R counts this CTA's ring uses; the K and V rings advance together
      // (a QF k-block stage fills both, a key tile one of each).
      int R = 0;
      bool ok = true;
      auto ring_ph = [](int rr) { return ((uint32_t)(rr / NST) & 1u) ^ 1u; };
      for (int I = 0; I < n_items && ok; ++I) {
        const Item it = item_of(item_k(I));
        const int hx = it.h * D;
        if (!QF) {
          if (!(ok = tc::mbar_wait(q_empty, ((uint32_t)I & 1u) ^ 1u, abort_flag, p.status))) break;
          tc::mbar_expect_tx(q_full, (uint32_t)(L::KB * L::TILE));
          for (int kb = 0; kb < L::KB; ++kb)
            tc::tma_load_2d(smem + L::Q_OFF + kb * L::TILE, &tmQ, q_full, hx + 64 * kb, it.b * p.S + it.m0);
        } else {
          // z_q rows of the tile (K ring) and V_q[:, head] (V ring), KB
          // k-blocks of 64 per stage
          for (int sq = 0; sq < nqs && ok; ++sq) {
            const int rr = R + sq, st = rr % NST;
            if (!(ok = tc::mbar_wait(k_empty + st, ring_ph(rr), abort_flag, p.status))) break;
            if (!(ok = tc::mbar_wait(v_empty + st, ring_ph(rr), abort_flag, p.status))) break;
            const int nb = min(L::KB, p.nq - sq * L::KB);
            tc::mbar_expect_tx(k_full + st, (uint32_t)(nb * L::TILE));
            tc::mbar_expect_tx(v_full + st, (uint32_t)(nb * L::KB * 8192));
            for (int kb = 0; kb < nb; ++kb) {
              const int kq = sq * L::KB + kb;
              tc::tma_load_2d(smem + L::K_OFF + (st * L::KB + kb) * L::TILE, &tmQ, k_full + st, kq * 64,
                              it.b * p.S + it.m0);
              uint8_t* vdst = smem + L::V_OFF + st * L::KB * L::TILE + kb * L::KB * 8192;
              for (int j = 0; j < L::KB; ++j)
                tc::tma_load_2d(vdst + j * 8192, &tmVq, v_full + st, hx + 64 * j, kq * 64);
            }
          }
          if (!ok) break;
          R += nqs;
        }
        // key tiles: K(0), then K(j + 1) before V(j)
        const int row0 = it.b * p.S_max;
        auto load_k = [&](int j) {
          const int rr = R + j, st = rr % NST;
          if (!tc::mbar_wait(k_empty + st, ring_ph(rr), abort_flag, p.status)) return false;
          tc::mbar_expect_tx(k_full + st, (uint32_t)(L::KB * L::TILE));
          for (int kb = 0; kb < L::KB; ++kb)
            tc::tma_load_2d(smem + L::K_OFF + (st * L::KB + kb) * L::TILE, &tmK, k_full + st, hx + 64 * kb,
                            row0 + j * AT_BN);
          return true;
        };
        auto load_v = [&](int j) {
          const int rr = R + j, st = rr % NST;
          if (!tc::mbar_wait(v_empty + st, ring_ph(rr), abort_flag, p.status)) return false;
          tc::mbar_expect_tx(v_full + st, (uint32_t)(L::KB * L::TILE));
          for (int kb = 0; kb < L::KB; ++kb)
            tc::tma_load_2d(smem + L::V_OFF + (st * L::KB + kb) * L::TILE, &tmV, v_full + st, hx + 64 * kb,
                            row0 + j * AT_BN);
          return true;
        };
        if (it.nt > 0) ok = load_k(0);
        for (int j = 0; j < it.nt && ok; ++j) {
          if (j + 1 < it.nt) ok = load_k(j + 1);
          ok = ok && load_v(j);
        }
        R += it.nt;
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t IDESC_S = tc::idesc_bf16(AT_BN, false);  // B = K rows, K-major
      constexpr uint32_t IDESC_O = tc::idesc_bf16(D, true);       // B = V rows, MN-major
      const uint32_t sq = tc::smem_u32(smem + L::Q_OFF);
      bool ok = true;
      int T = 0;  // S tiles of this CTA (S and P buffers, their barriers)
      int R = 0;  // ring uses of this CTA
      auto ring_ph = [](int rr) { return (uint32_t)(rr / NST) & 1u; };
      for (int I = 0; I < n_items && ok; ++I) {
        const Item it = item_of(item_k(I));
        // O (+)= P_t V_t once the softmax has written P_t (and rescaled O);
        // an item's first P V overwrites O, so the previous item's epilogue
        // must have read it.  V_t sits in V ring stage rr % NST.
        auto issue_pv = [&](int t, int rr, bool first) {
          const int pb = t & 1, st = rr % NST;
          if (!tc::mbar_wait(p_full + pb, (uint32_t)(t >> 1) & 1u, abort_flag, p.status)) return false;
          if (!tc::mbar_wait(v_full + st, ring_ph(rr), abort_flag, p.status)) return false;
          if (first && !tc::mbar_wait(o_free, ((uint32_t)I & 1u) ^ 1u, abort_flag, p.status)) return false;
          tc::fence_after_sync();
          const uint32_t sv = tc::smem_u32(smem + L::V_OFF + st * L::KB * L::TILE);
#pragma unroll
          for (int kk = 0; kk < AT_BN / 16; ++kk) {
            const uint64_t bd = tc::sdesc_sw128(sv + kk * 2048, L::TILE, 1024);
            tc::mma_bf16_ts(tmem + AT_TM_O, tmem + AT_TM_P + pb * 64 + kk * 8, bd, IDESC_O,
                            (!first || kk > 0) ? 1u : 0u);
          }
          tc::mma_commit(o_done + pb);
          tc::mma_commit(v_empty + st);
          return true;
        };
        if (QF) {
          // Q = z_q V_q[:, head] into TMEM columns 384.. (over the P
          // buffers) once the softmax warps have read the previous item's Q
          // and the previous item's last P V has read its P
          if (!(ok = tc::mbar_wait(qacc_free, ((uint32_t)I & 1u) ^ 1u, abort_flag, p.status))) break;
          if (T > 0 && !(ok = tc::mbar_wait(o_done + ((T - 1) & 1), (uint32_t)((T - 1) >> 1) & 1u, abort_flag,
                                            p.status)))
            break;
          for (int sq2 = 0; sq2 < nqs && ok; ++sq2) {
            const int rr = R + sq2, st = rr % NST;
            if (!(ok = tc::mbar_wait(k_full + st, ring_ph(rr), abort_flag, p.status))) break;
            if (!(ok = tc::mbar_wait(v_full + st, ring_ph(rr), abort_flag, p.status))) break;
            tc::fence_after_sync();
            const int nb = min(L::KB, p.nq - sq2 * L::KB);
            for (int kb = 0; kb < nb; ++kb) {
              const int kq = sq2 * L::KB + kb;
              const uint32_t sz = tc::smem_u32(smem + L::K_OFF + (st * L::KB + kb) * L::TILE);
              const uint32_t svq = tc::smem_u32(smem + L::V_OFF + st * L::KB * L::TILE + kb * L::KB * 8192);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = tc::sdesc_sw128(sz + kk * 32, 16, 1024);
                const uint64_t bd = tc::sdesc_sw128(svq + kk * 2048, 8192, 1024);
                tc::mma_bf16(tmem + AT_TM_P, ad, bd, IDESC_O, (kq > 0 || kk > 0) ? 1u : 0u);
              }
            }
            tc::mma_commit(k_empty + st);
            tc::mma_commit(v_empty + st);
          }
          if (!ok) break;
          R += nqs;
          tc::mma_commit(qacc_full);
        }
        if (!(ok = tc::mbar_wait(q_full, (uint32_t)I & 1u, abort_flag, p.status))) break;
        for (int j = 0; j < it.nt && ok; ++j) {
          const int t = T + j, sb = t & 1;
          const int rr = R + j, st = rr % NST;
          if (!(ok = tc::mbar_wait(k_full + st, ring_ph(rr), abort_flag, p.status))) break;
          if (!(ok = tc::mbar_wait(s_empty + sb, ((uint32_t)(t >> 1) & 1u) ^ 1u, abort_flag, p.status))) break;
          tc::fence_after_sync();
          const uint32_t sk = tc::smem_u32(smem + L::K_OFF + st * L::KB * L::TILE);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = tc::sdesc_sw128(sq + (kk >> 2) * L::TILE + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = tc::sdesc_sw128(sk + (kk >> 2) * L::TILE + (kk & 3) * 32, 16, 1024);
            tc::mma_bf16(tmem + sb * AT_BN, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
          }
          tc::mma_commit(s_full + sb);
          tc::mma_commit(k_empty + st);
          if (j > 0) ok = issue_pv(t - 1, rr - 1, j == 1);
        }
        if (!ok) break;
        tc::mma_commit(q_empty);  // fires once this item's S MMAs are done
        if (it.nt > 0) ok = issue_pv(T + it.nt - 1, R + it.nt - 1, it.nt == 1);
        T += it.nt;
        R += it.nt;
      }
      // every MMA this thread issued has completed once `drain` fires
      tc::mma_commit(drain);
      const long long t0 = clock64();
      while (!tc::mbar_try_wait(drain, 0) && clock64() - t0 < tc::kWaitCycles) {}
    }
  } else {
    // ------------------------------------------------- softmax, epilogue --
    // Warp w (2..9) reads TMEM lanes 32 (w % 4) .. + 31; warps 2-5 take keys
    // [0, 64) of a tile and O columns [0, D/2), warps 6-9 the other halves.
    // Both threads of a row read the whole row of S, so they take the same
    // row max (and the same rescale decisions) without an exchange.
    const int quad = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int r = quad * 32 + lane;       // query row within the tile
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    float* xr = reinterpret_cast<float*>(smem + L::X_OFF);  // [2 halves][128]
    const float sc = p.scale_log2;
    float m, l;                           // m: reference max, scaled units
    constexpr int HC = AT_BN / 2;         // keys per thread
    constexpr int OC = D / 2;             // O columns per thread
    // tcgen05.ld / st are warp-collective: wait results are made
    // warp-uniform.  The 8 softmax warps meet at a named barrier every
    // item, so the loop never exits early: after a failed wait it runs on
    // without touching tensor memory.
    auto wwait = [&](uint64_t* bar, uint32_t par) {
      return __all_sync(0xffffffffu, tc::mbar_wait(bar, par, abort_flag, p.status)) != 0;
    };
    auto sm_sync = [] { asm volatile("bar.sync 1, 256;" ::: "memory"); };
    bool ok = true;
    int T = 0;
    // (every item and tile is visited even after a failed wait, so that the
    // named barriers stay matched)
    for (int I = 0; I < n_items; ++I) {
    const Item it = item_of(item_k(I));
    const int m0 = it.m0, nt = it.nt, b = it.b, h = it.h;
    const int q = m0 + r;                 // query position
    m = -INFINITY;
    l = 0.f;
    if (QF) {
      // Q row r from TMEM: this thread rotates pairs (i, i + D/2) for
      // i in [hf D/4, (hf + 1) D/4) (rotate-half RoPE at position q) and
      // writes them as bf16 into the swizzled Q operand.
      constexpr int PQ = D / 4;
      const int base0 = D == 128 ? hf * 32 : 0;   // first column of the 32-column load
      ok = ok && wwait(qacc_full, (uint32_t)I & 1u);
      uint32_t qa[32], qb[32];
      if (ok) {
        tc::fence_after_sync();
        tc::tmem_ld32(tmem + lane_base + AT_TM_P + base0, qa);
        tc::tmem_ld32(tmem + lane_base + AT_TM_P + base0 + D / 2, qb);
        tc::tmem_ld_wait();
        tc::reg_fence<32>(qa);
        tc::reg_fence<32>(qb);
        if (p.zcnt && warp == 2) {
          // every Q MMA of this item has completed, so every TMA read of
          // its z_q rows is done; the last of the H heads' items drops the
          // rows' L2 lines without write-back (whole lines inside them)
          const int blk = b * qtiles + m0 / AT_BM;
          int last = 0;
          if (lane == 0) {
            last = atomicAdd(p.zcnt + blk, 1) == p.H - 1;
            if (last) p.zcnt[blk] = 0;
          }
          last = __shfl_sync(0xffffffffu, last, 0);
          if (last) {
            const long long b0 = ((long long)b * p.S + m0) * p.ldz * 2;
            const long long b1 = ((long long)b * p.S + min(m0 + AT_BM, p.S)) * p.ldz * 2;
            const uintptr_t zb = reinterpret_cast<uintptr_t>(p.zq);
            const uintptr_t l0 = (zb + b0 + 127) & ~(uintptr_t)127, l1 = (zb + b1) & ~(uintptr_t)127;
            for (uintptr_t ln = l0 + (uintptr_t)lane * 128; ln < l1; ln += 32 * 128)
              asm volatile("discard.global.L2 [%0], 128;" ::"l"(ln) : "memory");
          }
        }
      }
      // the previous item's S MMAs must be done before Q is rewritten
      ok = ok && wwait(q_empty, ((uint32_t)I & 1u) ^ 1u);
      if (ok) {
        const int i0 = hf * PQ;
        const bool valid = q < p.S;
        uint8_t* sQ = smem + L::Q_OFF;
#pragma unroll
        for (int ch = 0; ch < PQ / 8; ++ch) {
          float lo[8], hi[8];
#pragma unroll
          for (int u8 = 0; u8 < 8; ++u8) {
            const int e = ch * 8 + u8;
            // (i0 - base0 is 0 for D = 128 and hf * 16 for D = 64: both
            // registers are read and one selected, with constant indices)
            const uint32_t xa = (D == 64 && hf) ? qa[(e + 16) & 31] : qa[e];
            const uint32_t ya = (D == 64 && hf) ? qb[(e + 16) & 31] : qb[e];
            const float x = __uint_as_float(xa), y = __uint_as_float(ya);
            const float c = valid ? __ldg(p.rope_cos + (long long)q * (D / 2) + i0 + e) : 0.f;
            const float sn = valid ? __ldg(p.rope_sin + (long long)q * (D / 2) + i0 + e) : 0.f;
            lo[u8] = x * c - y * sn;
            hi[u8] = y * c + x * sn;
          }
#pragma unroll
          for (int half2 = 0; half2 < 2; ++half2) {
            const float* v = half2 ? hi : lo;
            const int col = half2 * (D / 2) + i0 + ch * 8;
            uint4 u;
            u.x = pack_bf2(v[0], v[1]); u.y = pack_bf2(v[2], v[3]);
            u.z = pack_bf2(v[4], v[5]); u.w = pack_bf2(v[6], v[7]);
            *reinterpret_cast<uint4*>(sQ + (col >> 6) * L::TILE + r * 128 + ((((col & 63) >> 3) ^ (r & 7)) << 4)) = u;
          }
        }
        tc::fence_proxy_async_smem();  // Q is read by the tensor cores
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(q_full);
        tc::mbar_arrive(qacc_free);
      }
    }
    for (int j = 0; j < nt; ++j) {
      const int t = T + j, sb = t & 1;
      // the P V of tile t - 2 must have read P buffer sb (checked first: it
      // has normally long completed)
      if (t >= 2) ok = ok && wwait(o_done + sb, (uint32_t)((t - 2) >> 1) & 1u);
      ok = ok && wwait(s_full + sb, (uint32_t)(t >> 1) & 1u);
      float s[HC], so[HC];  // this thread's half of the keys, the other half
      const bool masked = j * AT_BN + AT_BN > p.S || (CAUSAL && j * AT_BN + AT_BN - 1 > m0);
      const int n0 = j * AT_BN + hf * HC, n1 = j * AT_BN + (1 - hf) * HC;
      float mx8[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) mx8[c] = -INFINITY;
      if (ok) {
        tc::fence_after_sync();
        const uint32_t sa = tmem + lane_base + sb * AT_BN;
        // this thread's half first; its max runs while the other half loads
#pragma unroll
        for (int c = 0; c < HC / 32; ++c) tc::tmem_ld32(sa + hf * HC + c * 32, reinterpret_cast<uint32_t*>(s + c * 32));
        tc::tmem_ld_wait();
        tc::reg_fence<HC>(s);
#pragma unroll
        for (int c = 0; c < HC / 32; ++c)
          tc::tmem_ld32(sa + (1 - hf) * HC + c * 32, reinterpret_cast<uint32_t*>(so + c * 32));
        // mask (raw scores: the scale is positive) and row max
        if (masked) {
#pragma unroll
          for (int c = 0; c < HC; ++c)
            if (n0 + c >= p.S || (CAUSAL && n0 + c > q)) s[c] = -INFINITY;
        }
#pragma unroll
        for (int c = 0; c < HC; c += 2) mx8[(c >> 1) & 3] = max3(mx8[(c >> 1) & 3], s[c], s[c + 1]);
        tc::tmem_ld_wait();
        tc::reg_fence<HC>(so);
      } else {
#pragma unroll
        for (int c = 0; c < HC; ++c) s[c] = so[c] = -INFINITY;
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(s_empty + sb);
      if (masked) {
#pragma unroll
        for (int c = 0; c < HC; ++c)
          if (n1 + c >= p.S || (CAUSAL && n1 + c > q)) so[c] = -INFINITY;
      }
#pragma unroll
      for (int c = 0; c < HC; c += 2) mx8[4 + ((c >> 1) & 3)] = max3(mx8[4 + ((c >> 1) & 3)], so[c], so[c + 1]);
      const float rawmax = fmaxf(fmaxf(max3(mx8[0], mx8[1], mx8[2]), max3(mx8[3], mx8[4], mx8[5])),
                                 fmaxf(mx8[6], mx8[7]));
      const float mx = rawmax == -INFINITY ? -INFINITY : rawmax * sc;
      // The row's reference m (P = 2^(s sc - m)) moves up only when the tile
      // max exceeds it by more than 8: P stays <= 2^8 (exact enough in bf16
      // and in the fp32 sums), O and l keep the same reference, and O is
      // rescaled rarely.
      const bool raise = m == -INFINITY || mx > m + 8.f;
      const float m_new = raise ? fmaxf(mx, m) : m;
      const bool grow = j > 0 && raise && m != -INFINITY;
      if (ok && __any_sync(0xffffffffu, grow)) {
        // every P V so far (they complete in order) must be done
        ok = wwait(o_done + ((t - 1) & 1), (uint32_t)((t - 1) >> 1) & 1u);
        if (ok) {
          tc::fence_after_sync();
          const float corr = grow ? exp2f(m - m_new) : 1.f;
          l *= corr;
#pragma unroll
          for (int c = 0; c < OC / 32; ++c) {
            uint32_t o[32];
            tc::tmem_ld32(tmem + lane_base + AT_TM_O + hf * OC + c * 32, o);
            tc::tmem_ld_wait();
            tc::reg_fence<32>(o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
            tc::tmem_st32(tmem + lane_base + AT_TM_O + hf * OC + c * 32, o);
          }
          tc::tmem_st_wait();
        }
      }
      m = m_new;
      // P = 2^(s sc - m) as bf16 pairs into this half of P buffer sb
      const float mneg = m == -INFINITY ? 0.f : -m;
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[HC / 2];
#pragma unroll
      for (int e = 0; e < HC; e += 2) {
        float x0 = s[e], x1 = s[e + 1];
        fma2_sc(x0, x1, sc, mneg);  // masked keys: -inf, and 2^-inf = 0
        if (((e >> 1) & 3) < AT_EMU) {
          ex2_poly2(x0, x1);
        } else {
          x0 = ex2_approx(x0);
          x1 = ex2_approx(x1);
        }
        const float p0 = x0, p1 = x1;
        add2(l4[e & 3], l4[(e + 1) & 3], p0, p1);
        pk[e >> 1] = pack_bf2(p0, p1);
      }
      l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      if (ok) {
        tc::tmem_st32(tmem + lane_base + AT_TM_P + sb * 64 + hf * 32, pk);
        tc::tmem_st_wait();
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(p_full + sb);
    }
    // ---- O / l -> bf16 ----
    const int tl = T + nt - 1;
    const bool fin = ok && nt > 0 && wwait(o_done + (tl & 1), (uint32_t)(tl >> 1) & 1u);
    xr[hf * 128 + r] = l;
    sm_sync();
    const float lt = xr[r] + xr[128 + r];
    sm_sync();  // both halves have read l before the next item rewrites xr
    if (fin) {
      tc::fence_after_sync();
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const long long HD = (long long)p.H * D;
      bf16* og = p.out + ((long long)b * p.S + q) * HD + (long long)h * D + hf * OC;
#pragma unroll
      for (int c = 0; c < OC / 32; ++c) {
        uint32_t o[32];
        tc::tmem_ld32(tmem + lane_base + AT_TM_O + hf * OC + c * 32, o);
        tc::tmem_ld_wait();
        tc::reg_fence<32>(o);
        if (q < p.S) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 u;
            u.x = pack_bf2(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv);
            u.y = pack_bf2(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
            u.z = pack_bf2(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
            u.w = pack_bf2(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
            *reinterpret_cast<uint4*>(og + c * 32 + e) = u;
          }
        }
      }
    }
    // O is read: the next item's first P V may overwrite it
    tc::fence_before_sync();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(o_free);
    T += nt;
    }  // items
  }

  tc::fence_before_sync();
  __syncthreads();
  if (*abort_flag && warp == 0 && lane == 0) {
    // let copies still in flight land before shared memory is released
    const long long t0 = clock64();
    while (clock64() - t0 < 2000000) {}
  }
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512);
  }
}

template <int D, bool CAUSAL, bool QF>
int launch_at(const AttnPfParams& ap, cudaStream_t stream) {
  using L = AtLayout<D>;
  auto kern = attn_prefill_tc_kernel<D, CAUSAL, QF>;
  static SmemAttrOnce smem_once;
  FSVD_TRY(set_smem_once(smem_once, kern, L::SMEM));
  const long long HD = (long long)ap.H * D;
  CUtensorMap mq, mk, mv, mvq;
  if (QF) {
    FSVD_TRY(encode_map(&mq, ap.zq, (long long)ap.B * ap.S, ap.r, ap.ldz, 64, AT_BM, true));
    FSVD_TRY(encode_map(&mvq, ap.Vq, ap.r, HD, HD, 64, 64, true));
  } else {
    FSVD_TRY(encode_map(&mq, ap.q, (long long)ap.B * ap.S, HD, HD, 64, AT_BM, true));
    mvq = mq;  // unused
  }
  FSVD_TRY(encode_map(&mk, ap.k, (long long)ap.B * ap.S_max, HD, HD, 64, AT_BN, true));
  FSVD_TRY(encode_map(&mv, ap.v, (long long)ap.B * ap.S_max, HD, HD, 64, AT_BN, true));
  AtParams p;
  memset(&p, 0, sizeof(p));
  p.B = ap.B; p.S = ap.S; p.H = ap.H; p.S_max = ap.S_max;
  p.scale_log2 = ap.scale_log2;
  p.out = ap.out;
  p.status = ap.status;
  const int qtiles = ceil_div(ap.S, AT_BM);
  if (QF) {
    p.nq = ap.r / 64;
    p.zq = ap.zq; p.ldz = ap.ldz;
    p.rope_cos = ap.rope_cos; p.rope_sin = ap.rope_sin;
    p.zcnt = (ap.zcnt && (long long)ap.B * qtiles <= ap.zcnt_cap) ? ap.zcnt : nullptr;
  }
  const int items = qtiles * ap.B * ap.H;
  int sms = 148;
  {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  }
  const dim3 grid(items < sms ? items : sms);
  const double S = ap.S;
  double flops = 4.0 * ap.B * ap.H * S * S * D * (CAUSAL ? 0.5 : 1.0);
  double bytes = 2.0 * 4.0 * ap.B * S * HD;
  if (QF) {
    flops += 2.0 * ap.B * S * (double)ap.r * HD;            // Q = z_q V_q
    bytes += 2.0 * ((double)ap.B * S * ap.r + (double)ap.r * HD) - 2.0 * ap.B * S * HD;  // z_q, V_q for q
  }
  const char* name = QF ? (CAUSAL ? "attn_prefill_causal_qf" : "attn_prefill_bidir_qf")
                        : (CAUSAL ? "attn_prefill_causal" : "attn_prefill_bidir");
  const LaunchTag tag{name, bytes, flops};
  return launch_pdl(tag, kern, grid, dim3(AT_THREADS), (size_t)L::SMEM, stream, mq, mk, mv, mvq, p);
}

}  // namespace

int attn_prefill_launch(const AttnPfParams& p, cudaStream_t stream) {
  if (!p.status) return FLASHSVD_ERR_NOT_INITIALIZED;
  if (p.zq) {
    if (!p.Vq || !p.rope_cos || !p.rope_sin || p.r <= 0 || p.r % 64) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
    if (p.D == 128) return p.causal ? launch_at<128, true, true>(p, stream) : launch_at<128, false, true>(p, stream);
    if (p.D == 64) return p.causal ? launch_at<64, true, true>(p, stream) : launch_at<64, false, true>(p, stream);
    return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  }
  if (p.D == 128) return p.causal ? launch_at<128, true, false>(p, stream) : launch_at<128, false, false>(p, stream);
  if (p.D == 64) return p.causal ? launch_at<64, true, false>(p, stream) : launch_at<64, false, false>(p, stream);
  return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace fsvd
