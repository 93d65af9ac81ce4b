// Prefill attention on the 5th-generation tensor cores.
//
// FlashSVD v1.5 (gist.science explainer), Technical Summary, Methodology 2:
// prefill keeps its own attention kernel (the dense-KV path is the decode
// one); here it reads the same dense [B, S_max, H, D] cache the prefill's
// q/k/v epilogue wrote.  Causal (decoder) or bidirectional (encoder).
//
// Persistent CTAs (one per SM) walk the (128-query tile, batch row, head)
// items, heaviest first; 10 warps:
//   warp 0  TMA: Q once, then 128-key K and V tiles into a 2-stage ring;
//   warp 1  TMEM owner and MMA issuer: S = Q K^T into one of two 128-column
//           TMEM buffers, then O += P V into a D-column TMEM accumulator;
//   warps 2-9  two threads per query row (each half of the keys and of O):
//           load S from TMEM, mask, online softmax (exp2 domain, the row max
//           exchanged through shared memory), rescale O in TMEM when the
//           row's reference max moves, write P (bf16) into 128-byte-swizzled
//           shared memory as the next MMA's A operand; at the end O / l.
// All operand tiles are 128-byte swizzled; S of tile j+1 is computed while
// the softmax of tile j runs.  Every wait is bounded.
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
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + KB * TILE;
  static constexpr int V_OFF = K_OFF + 2 * KB * TILE;
  static constexpr int P_OFF = V_OFF + 2 * KB * TILE;
  static constexpr int BAR_OFF = P_OFF + 2 * TILE;
  static constexpr int X_OFF = BAR_OFF + 256;     // [2 tiles][2 halves][128] row partials
  static constexpr int SMEM = 1024 + X_OFF + 2 * 2 * 128 * 4;
  static_assert(SMEM <= 232448, "shared memory budget");
};

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
  uint64_t* q_full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* kv_full = q_full + 1;    // [2]
  uint64_t* kv_empty = kv_full + 2;  // [2]
  uint64_t* s_full = kv_empty + 2;   // [2]
  uint64_t* s_empty = s_full + 2;    // [2]
  uint64_t* p_full = s_empty + 2;
  uint64_t* o_done = p_full + 1;
  uint64_t* drain = o_done + 1;
  uint64_t* q_empty = drain + 1;     // the item's S MMAs are done: Q may be reloaded
  uint64_t* o_free = q_empty + 1;    // the epilogue has read O (count 8)
  uint64_t* qacc_full = o_free + 1;  // QF: the item's Q = z_q V_q is in TMEM
  uint64_t* qacc_free = qacc_full + 1;  // QF: the softmax warps have read it (count 8)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(qacc_free + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Persistent: work item k = (query tile, batch row, head), heaviest
  // (longest causal) query tiles first; CTA c takes items c, c + G, ...
  // Barrier phases run on across items: T counts this CTA's key tiles, I
  // its items.
  const int qtiles = (p.S + AT_BM - 1) / AT_BM;
  const int BH = p.B * p.H;
  const int NW = qtiles * BH;
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
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(kv_full + i, 1);
      tc::mbar_init(kv_empty + i, 1);
      tc::mbar_init(s_full + i, 1);
      tc::mbar_init(s_empty + i, 8);
    }
    tc::mbar_init(p_full, 8);
    tc::mbar_init(o_done, 1);
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
    tc::tmem_alloc(tmem_holder, 512);  // S0 [0,128), S1 [128,256), O [256, 256 + D), QF: Q [384, 384 + D)
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
      int R = 0;  // ring uses of this CTA (K/V tiles, and QF's z_q / V_q k-blocks)
      bool ok = true;
      for (int k = blockIdx.x, I = 0; k < NW && ok; k += gridDim.x, ++I) {
        const Item it = item_of(k);
        const int hx = it.h * D;
        if (!QF) {
          if (!(ok = tc::mbar_wait(q_empty, ((uint32_t)I & 1u) ^ 1u, abort_flag, p.status))) break;
          tc::mbar_expect_tx(q_full, (uint32_t)(L::KB * L::TILE));
          for (int kb = 0; kb < L::KB; ++kb)
            tc::tma_load_2d(smem + L::Q_OFF + kb * L::TILE, &tmQ, q_full, hx + 64 * kb, it.b * p.S + it.m0);
        } else {
          // z_q rows of the tile (K region) and V_q[:, head] (V region), KB
          // k-blocks of 64 per ring stage
          for (int sq = 0; sq < nqs && ok; ++sq) {
            const int rr = R + sq, st = rr & 1;
            if (!(ok = tc::mbar_wait(kv_empty + st, ((uint32_t)(rr >> 1) & 1u) ^ 1u, abort_flag, p.status))) break;
            const int nb = min(L::KB, p.nq - sq * L::KB);
            tc::mbar_expect_tx(kv_full + st, (uint32_t)(nb * (L::TILE + L::KB * 8192)));
            for (int kb = 0; kb < nb; ++kb) {
              const int kq = sq * L::KB + kb;
              tc::tma_load_2d(smem + L::K_OFF + (st * L::KB + kb) * L::TILE, &tmQ, kv_full + st, kq * 64,
                              it.b * p.S + it.m0);
              uint8_t* vdst = smem + L::V_OFF + st * L::KB * L::TILE + kb * L::KB * 8192;
              for (int j = 0; j < L::KB; ++j)
                tc::tma_load_2d(vdst + j * 8192, &tmVq, kv_full + st, hx + 64 * j, kq * 64);
            }
          }
          if (!ok) break;
          R += nqs;
        }
        for (int j = 0; j < it.nt; ++j) {
          const int t = R + j, st = t & 1;
          if (!(ok = tc::mbar_wait(kv_empty + st, ((uint32_t)(t >> 1) & 1u) ^ 1u, abort_flag, p.status))) break;
          tc::mbar_expect_tx(kv_full + st, (uint32_t)(2 * L::KB * L::TILE));
          const int row = it.b * p.S_max + j * AT_BN;
          for (int kb = 0; kb < L::KB; ++kb) {
            tc::tma_load_2d(smem + L::K_OFF + (st * L::KB + kb) * L::TILE, &tmK, kv_full + st, hx + 64 * kb, row);
            tc::tma_load_2d(smem + L::V_OFF + (st * L::KB + kb) * L::TILE, &tmV, kv_full + st, hx + 64 * kb, row);
          }
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
      const uint32_t sp = tc::smem_u32(smem + L::P_OFF);
      bool ok = true;
      int T = 0;  // S tiles of this CTA (S buffers, P, O barriers)
      int R = 0;  // ring uses of this CTA
      for (int k = blockIdx.x, I = 0; k < NW && ok; k += gridDim.x, ++I) {
        const Item it = item_of(k);
        // O (+)= P_t V_t once the softmax has written P_t (and rescaled O);
        // an item's first P V overwrites O, so the previous item's epilogue
        // must have read it.  V_t sits in ring stage rr & 1.
        auto issue_pv = [&](int t, int rr, bool first) {
          if (!tc::mbar_wait(p_full, (uint32_t)t & 1u, abort_flag, p.status)) return false;
          if (first && !tc::mbar_wait(o_free, ((uint32_t)I & 1u) ^ 1u, abort_flag, p.status)) return false;
          tc::fence_after_sync();
          const uint32_t sv = tc::smem_u32(smem + L::V_OFF + (rr & 1) * L::KB * L::TILE);
#pragma unroll
          for (int kk = 0; kk < AT_BN / 16; ++kk) {
            const uint64_t ad = tc::sdesc_sw128(sp + (kk >> 2) * L::TILE + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = tc::sdesc_sw128(sv + kk * 2048, L::TILE, 1024);
            tc::mma_bf16(tmem + 256, ad, bd, IDESC_O, (!first || kk > 0) ? 1u : 0u);
          }
          tc::mma_commit(o_done);
          tc::mma_commit(kv_empty + (rr & 1));
          return true;
        };
        if (QF) {
          // Q = z_q V_q[:, head] into TMEM columns 384.. once the softmax
          // warps have read the previous item's Q
          if (!(ok = tc::mbar_wait(qacc_free, ((uint32_t)I & 1u) ^ 1u, abort_flag, p.status))) break;
          for (int sq = 0; sq < nqs && ok; ++sq) {
            const int rr = R + sq, st = rr & 1;
            if (!(ok = tc::mbar_wait(kv_full + st, (uint32_t)(rr >> 1) & 1u, abort_flag, p.status))) break;
            tc::fence_after_sync();
            const int nb = min(L::KB, p.nq - sq * L::KB);
            for (int kb = 0; kb < nb; ++kb) {
              const int kq = sq * L::KB + kb;
              const uint32_t sz = tc::smem_u32(smem + L::K_OFF + (st * L::KB + kb) * L::TILE);
              const uint32_t svq = tc::smem_u32(smem + L::V_OFF + st * L::KB * L::TILE + kb * L::KB * 8192);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = tc::sdesc_sw128(sz + kk * 32, 16, 1024);
                const uint64_t bd = tc::sdesc_sw128(svq + kk * 2048, 8192, 1024);
                tc::mma_bf16(tmem + 384, ad, bd, IDESC_O, (kq > 0 || kk > 0) ? 1u : 0u);
              }
            }
            tc::mma_commit(kv_empty + st);
          }
          if (!ok) break;
          R += nqs;
          tc::mma_commit(qacc_full);
        }
        if (!(ok = tc::mbar_wait(q_full, (uint32_t)I & 1u, abort_flag, p.status))) break;
        for (int j = 0; j < it.nt && ok; ++j) {
          const int t = T + j, st = t & 1;
          const int rr = R + j, sr = rr & 1;
          if (!(ok = tc::mbar_wait(kv_full + sr, (uint32_t)(rr >> 1) & 1u, abort_flag, p.status))) break;
          if (!(ok = tc::mbar_wait(s_empty + st, ((uint32_t)(t >> 1) & 1u) ^ 1u, abort_flag, p.status))) break;
          tc::fence_after_sync();
          const uint32_t sk = tc::smem_u32(smem + L::K_OFF + sr * L::KB * L::TILE);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ad = tc::sdesc_sw128(sq + (kk >> 2) * L::TILE + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = tc::sdesc_sw128(sk + (kk >> 2) * L::TILE + (kk & 3) * 32, 16, 1024);
            tc::mma_bf16(tmem + st * AT_BN, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
          }
          tc::mma_commit(s_full + st);
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
    const int quad = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int r = quad * 32 + lane;       // query row within the tile
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    float* xr = reinterpret_cast<float*>(smem + L::X_OFF);  // [2][2][128]
    const float sc = p.scale_log2;
    float m, l;                           // m: reference max, scaled units
    uint8_t* sP = smem + L::P_OFF;
    constexpr int HC = AT_BN / 2;         // keys per thread
    constexpr int OC = D / 2;             // O columns per thread
    // tcgen05.ld / st are warp-collective: wait results are made
    // warp-uniform.  The 8 softmax warps meet at a named barrier every tile,
    // so the loop never exits early: after a failed wait it runs on without
    // touching tensor memory.
    auto wwait = [&](uint64_t* bar, uint32_t par) {
      return __all_sync(0xffffffffu, tc::mbar_wait(bar, par, abort_flag, p.status)) != 0;
    };
    auto sm_sync = [] { asm volatile("bar.sync 1, 256;" ::: "memory"); };
    bool ok = true;
    int T = 0;
    // (every item and tile is visited even after a failed wait, so that the
    // named barriers stay matched)
    for (int k = blockIdx.x, I = 0; k < NW; k += gridDim.x, ++I) {
    const Item it = item_of(k);
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
        tc::tmem_ld32(tmem + lane_base + 384 + base0, qa);
        tc::tmem_ld32(tmem + lane_base + 384 + base0 + D / 2, qb);
        tc::tmem_ld_wait();
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
      const int t = T + j, st = t & 1;
      ok = ok && wwait(s_full + st, (uint32_t)(t >> 1) & 1u);
      float s[HC];
      if (ok) {
        tc::fence_after_sync();
#pragma unroll
        for (int c = 0; c < HC / 32; ++c)
          tc::tmem_ld32(tmem + lane_base + st * AT_BN + hf * HC + c * 32, reinterpret_cast<uint32_t*>(s + c * 32));
        tc::tmem_ld_wait();
      } else {
#pragma unroll
        for (int c = 0; c < HC; ++c) s[c] = -INFINITY;
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(s_empty + st);
      // mask (raw scores: the scale is positive) and partial row max
      const int n0 = j * AT_BN + hf * HC;
      const bool need_mask = n0 + HC > p.S || (CAUSAL && n0 + HC - 1 > m0);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < HC; ++c) {
          const int key = n0 + c;
          if (key >= p.S || (CAUSAL && key > q)) s[c] = -INFINITY;
        }
      }
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < HC; c += 2) mx4[(c >> 1) & 3] = max3(mx4[(c >> 1) & 3], s[c], s[c + 1]);
      float* xt = xr + st * 256;
      xt[hf * 128 + r] = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      sm_sync();
      const float rawmax = fmaxf(xt[r], xt[128 + r]);
      const float mx = rawmax == -INFINITY ? -INFINITY : rawmax * sc;
      // PV of tile j-1 must be complete before O is rescaled or P rewritten
      if (j > 0) ok = ok && wwait(o_done, (uint32_t)(t - 1) & 1u);
      tc::fence_after_sync();
      // The row's reference m (P = 2^(s sc - m)) moves up only when the tile
      // max exceeds it by more than 8: P stays <= 2^8 (exact enough in bf16
      // and in the fp32 sums), O and l keep the same reference, and O is
      // rescaled rarely.
      const bool raise = m == -INFINITY || mx > m + 8.f;
      const float m_new = raise ? fmaxf(mx, m) : m;
      const bool grow = j > 0 && raise && m != -INFINITY;
      if (ok && __any_sync(0xffffffffu, grow)) {
        const float corr = grow ? exp2f(m - m_new) : 1.f;
        l *= corr;
#pragma unroll
        for (int c = 0; c < OC / 32; ++c) {
          uint32_t o[32];
          tc::tmem_ld32(tmem + lane_base + 256 + hf * OC + c * 32, o);
          tc::tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
          tc::tmem_st32(tmem + lane_base + 256 + hf * OC + c * 32, o);
        }
        tc::tmem_st_wait();
      }
      m = m_new;
      // P = 2^(s sc - m), bf16, this half of row r of the swizzled A operand
      const float mneg = m == -INFINITY ? 0.f : -m;
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ch = 0; ch < HC / 8; ++ch) {
        float pv[8];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          float x0 = s[ch * 8 + e], x1 = s[ch * 8 + e + 1];
          fma2_sc(x0, x1, sc, mneg);  // masked keys: -inf, and 2^-inf = 0
          pv[e] = ex2_approx(x0);
          pv[e + 1] = ex2_approx(x1);
          add2(l4[e & 3], l4[(e + 1) & 3], pv[e], pv[e + 1]);
        }
        uint4 u;
        u.x = pack_bf2(pv[0], pv[1]); u.y = pack_bf2(pv[2], pv[3]);
        u.z = pack_bf2(pv[4], pv[5]); u.w = pack_bf2(pv[6], pv[7]);
        *reinterpret_cast<uint4*>(sP + hf * L::TILE + r * 128 + ((ch ^ (r & 7)) << 4)) = u;
      }
      l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      tc::fence_proxy_async_smem();   // P is read by the tensor cores
      tc::fence_before_sync();        // O rows rewritten in TMEM above
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(p_full);
    }
    // ---- O / l -> bf16 ----
    const bool fin = ok && nt > 0 && wwait(o_done, (uint32_t)(T + nt - 1) & 1u);
    sm_sync();  // every partner has read the last tile's row maxima
    xr[hf * 128 + r] = l;
    sm_sync();
    const float lt = xr[r] + xr[128 + r];
    sm_sync();  // both halves have read l before the next item's maxima reuse xr
    if (fin) {
      tc::fence_after_sync();
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const long long HD = (long long)p.H * D;
      bf16* og = p.out + ((long long)b * p.S + q) * HD + (long long)h * D + hf * OC;
#pragma unroll
      for (int c = 0; c < OC / 32; ++c) {
        uint32_t o[32];
        tc::tmem_ld32(tmem + lane_base + 256 + hf * OC + c * 32, o);
        tc::tmem_ld_wait();
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
