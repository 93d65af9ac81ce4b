// Fused decode layer: the whole decode step of one low-rank decoder layer in
// one persistent kernel (one CTA per SM).
//
// FlashSVD v1.5 (gist.science explainer), Technical Summary: decode is
// memory-bound (Problem Statement), the present token's q/k/v are rebuilt
// through the low-rank projections and the history is read from a dense KV
// cache (Methodology 2), gate and up share one packed projection
// (Methodology 3), and the per-layer decode body is one replay unit
// (Methodology 4).  Here that replay unit is a single kernel whose nine
// stages (z = rmsnorm(x) U_qkv; q,k,v = z V (+RoPE, KV append); attention;
// z = a U_o; x += z V_o; z = rmsnorm(x) U_gu; h = SiLU(z_g V_g) (z_u V_u);
// z = h U_dn; x += z V_dn) are separated by grid barriers, while the bytes
// that do not depend on any stage -- every factor tile -- stream without
// pause.
//
// The factors are read from the layer's decode pack: every factor matrix
// re-tiled once, at load time, so that each ring entry (256 rows x 64
// output columns, as two [rows x 32] boxes) is one contiguous block of HBM,
// stored in the order the stages consume them.  Streaming whole blocks
// instead of 64- or 128-byte row pieces scattered at the matrix's row pitch
// is what lets the factor stream run near the HBM roofline.
//
// Roles per CTA (CW consumer warps + 2 producer warps):
//   warp CW   factor producer: walks this CTA's schedule across all stages and
//             bulk-copies each entry of the pack into a ring slot as soon as
//             the slot is free (and prefetches the next entries into L2); it
//             never waits for activations.
//   warp CW+1 activation producer: after each stage's grid barrier, bulk-copies
//           the activation rows each ring entry needs (and, for attention,
//           the K/V chunk) into the same slot.
//   warps 0..CW-1 consumers: multiply, keep whole K ranges in registers, and
//           finish a column tile either directly (sole owner) or through a
//           last-arriver combine of per-CTA partials (fixed order).
// A CTA's share of a stage is a contiguous range of (tile, 256-row chunk)
// entries, so partial sums are written once per tile touched (1-4 per stage)
// instead of once per chunk.  All waits are bounded.
#include <algorithm>
#include <cstring>

#include "kernels.h"
#include "tc.cuh"

namespace fsvd {

namespace {

constexpr int DF_KC = 256;
constexpr int DF_MAX_SU = 16;
constexpr int DF_PART_STRIDE = 640;
constexpr int DF_NPHASE = 9;
constexpr int DF_NMAPS = 2;

enum { DF_GEMV = 0, DF_ATTN = 1 };

struct DfPhase {
  int type, pro, epi, map;
  int nprob;
  int tile_start[4];
  int T, K, nk;
  long long pack_off;  // byte offset of this stage's entries in the pack
  int N[3];
  int a_col[3];
  int a_col2;
  int w_row2;
  int out_col[3];
  int kind[3];
  const void* a;
  int a_f32;
  long long lda;
  const bf16* norm_g;
  float* out32; long long ldo32;
  bf16* out16; long long ldo16;
  const bf16* resid; long long ldr;
};

struct DfParams {
  CUtensorMap maps[DF_NMAPS];  // the K and V cache views [B * S_max x H * D]
  const uint8_t* pack;
  DfPhase ph[DF_NPHASE];
  int nphase;
  int B, H, D, S_max;
  float eps, scale_log2;
  const int* seqlens;
  bf16* k_cache;
  bf16* v_cache;
  const float* rope_cos;
  const float* rope_sin;
  const bf16* q;
  bf16* att;
  float* part;
  int* tilecnt;
  int* bar;
  int* done;
  int* status;
};

template <int MT>
struct DfCfg {
  static constexpr int CW = MT <= 2 ? 16 : 8;        // consumer warps
  static constexpr int CT = CW * 32;                 // consumer threads
  static constexpr int THREADS = CT + 64;            // + factor and activation producers
  static constexpr int W_BYTES = 32768;
  static constexpr int A_BYTES = 2 * MT * DF_KC * 4;
  static constexpr int SLOT = W_BYTES + A_BYTES;
  static constexpr int NSLOT = MT == 1 ? 6 : (MT == 8 ? 4 : 5);
  static constexpr int RED_BYTES = CW * MT * 64 * 4 > 2048 ? CW * MT * 64 * 4 : 2048;
  static constexpr int SCR_BYTES = (64 + CW * 128 + 128) * 4;
  static constexpr int BAR_BYTES = 1024;
  static constexpr int PH_BYTES = 2048;  // copy of the stage table
  static constexpr int SMEM = 1024 + NSLOT * SLOT + RED_BYTES + SCR_BYTES + BAR_BYTES + PH_BYTES;
  static_assert(SMEM <= 232448, "shared memory budget");
};

template <int N>
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void prefetch_l2_bulk(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          tc::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect(uint64_t* bar, uint32_t bytes) {
  tc::mbar_expect_tx(bar, bytes);  // arrive (count 1) + expect bytes
}
__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Contiguous share [c0, c1) of C entries for CTA g of G; owner of entry c.
// (32-bit: C * G stays below 2^31 for every stage the host accepts.)
__device__ __forceinline__ void share(int C, int G, int g, int& c0, int& c1) {
  c0 = g * C / G;
  c1 = (g + 1) * C / G;
}
__device__ __forceinline__ int owner_of(int c, int C, int G) {
  return ((c + 1) * G - 1) / C;
}

// Whether CTA g has at least one of the C entries.
__device__ __forceinline__ bool share_nonempty(int C, int G, int g) {
  return (g + 1) * C / G > g * C / G;
}
// Number of distinct CTAs owning entries first..last: every CTA between the
// two owners when each CTA has entries (C >= G), else only the non-empty ones.
__device__ __forceinline__ int count_owners(int first, int last, int C, int G) {
  const int gf = owner_of(first, C, G), gl = owner_of(last, C, G);
  if (C >= G) return gl - gf + 1;
  int n = 0;
  for (int gg = gf; gg <= gl; ++gg) n += share_nonempty(C, G, gg);
  return n;
}

// Attention entry layout: for each batch row b, H heads x nk_b chunks of 64
// keys (nk_b from the current length).
struct AttnSched {
  int nk[8];
  int pre[9];
  int L[8];
};
__device__ __forceinline__ void attn_sched(const DfParams& p, AttnSched& s) {
  s.pre[0] = 0;
  for (int b = 0; b < 8; ++b) {
    if (b < p.B) {
      int pos = p.seqlens[b];
      pos = pos < 0 ? 0 : (pos >= p.S_max ? p.S_max - 1 : pos);
      s.L[b] = pos + 1;
      s.nk[b] = (s.L[b] + 63) / 64;
    } else {
      s.L[b] = 0;
      s.nk[b] = 0;
    }
    s.pre[b + 1] = s.pre[b] + p.H * s.nk[b];
  }
}
__device__ __forceinline__ void attn_entry(const AttnSched& s, int c, int& b, int& h, int& kc) {
  b = 0;
  while (b < 7 && c >= s.pre[b + 1]) ++b;
  const int r = c - s.pre[b];
  h = r / s.nk[b];
  kc = r - h * s.nk[b];
}

// Global output column of tile column c (0..63).
__device__ __forceinline__ int out_col(const DfPhase& ph, int D, int tl, int c) {
  const int box = c >> 5, cc = c & 31;
  if (ph.map == MAP_PLAIN) return 64 * tl + c;
  if (ph.map == MAP_ROPE) {
    const int tph = D >> 6, hh = tl / tph, j = tl - hh * tph;
    return hh * D + 32 * j + cc + box * (D >> 1);
  }
  return 32 * tl + cc;
}

// acc[m][0..7] += A[m][kk] * W[kk][8 columns] over this thread's 8 rows of
// a 256-row entry.  NORM: A is bf16 x scaled by rstd[m] * g[kk]; AF32: A is
// fp32 (rank activations), else bf16.
template <int MT, int NORM, int AF32, int RSTEP>
__device__ __forceinline__ void entry_mac(float (&acc)[MT][8], const uint8_t* w, const uint8_t* a_s,
                                          int seg, int kn, int row0, const bf16* g,
                                          const float* rstd) {
  constexpr int IT = DF_KC / RSTEP;
  // All shared-memory loads of this thread's rows first (slots are always
  // fully allocated), then the arithmetic; rows at or beyond kn are masked.
  uint4 u[IT];
  float a[IT][MT];
#pragma unroll
  for (int i = 0; i < IT; ++i) {
    const int kk = row0 + RSTEP * i;
    u[i] = *reinterpret_cast<const uint4*>(w + kk * 64);
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (AF32) a[i][m] = reinterpret_cast<const float*>(a_s)[(seg * MT + m) * DF_KC + kk];
      else a[i][m] = bf2f(reinterpret_cast<const bf16*>(a_s)[(seg * MT + m) * DF_KC + kk]);
    }
  }
  float gk[IT];
#pragma unroll
  for (int i = 0; i < IT; ++i) {
    const int kk = row0 + RSTEP * i;
    gk[i] = NORM ? bf2f(g[kk < kn ? kk : 0]) : 1.f;
  }
#pragma unroll
  for (int i = 0; i < IT; ++i) {
    const bool valid = row0 + RSTEP * i < kn;
    const float wv[8] = {bf_lo(u[i].x), bf_hi(u[i].x), bf_lo(u[i].y), bf_hi(u[i].y),
                         bf_lo(u[i].z), bf_hi(u[i].z), bf_lo(u[i].w), bf_hi(u[i].w)};
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float av = NORM ? a[i][m] * (rstd[m] * gk[i]) : a[i][m];
      av = valid ? av : 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[m][j] = fmaf(av, valid ? wv[j] : 0.f, acc[m][j]);
    }
  }
}

template <int MT>
__global__ void __launch_bounds__(DfCfg<MT>::THREADS, 1)
decode_layer_kernel(const __grid_constant__ DfParams p) {
  using C = DfCfg<MT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* slots = smem;
  float* red = reinterpret_cast<float*>(smem + C::NSLOT * C::SLOT);
  float* scr = reinterpret_cast<float*>(smem + C::NSLOT * C::SLOT + C::RED_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::NSLOT * C::SLOT + C::RED_BYTES + C::SCR_BYTES);
  uint64_t* empty = full + C::NSLOT;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + C::NSLOT);
  int* s_flag = const_cast<int*>(abort_flag) + 1;
  float* s_rstd = reinterpret_cast<float*>(s_flag + 4);  // [8]
  DfPhase* s_ph = reinterpret_cast<DfPhase*>(smem + C::NSLOT * C::SLOT + C::RED_BYTES + C::SCR_BYTES +
                                             C::BAR_BYTES);
  static_assert(sizeof(DfPhase) * DF_NPHASE <= 2048, "stage table exceeds its shared-memory copy");

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, g = blockIdx.x;

  {
    // Stage descriptors are read in every inner loop: keep a shared copy.
    const int* src = reinterpret_cast<const int*>(p.ph);
    int* dst = reinterpret_cast<int*>(s_ph);
    for (int i = tid; i < (int)(sizeof(DfPhase) * DF_NPHASE / 4); i += C::THREADS) dst[i] = src[i];
  }
  if (tid == 0) {
    for (int s = 0; s < C::NSLOT; ++s) {
      tc::mbar_init(full + s, 2);
      tc::mbar_init(empty + s, C::CW);
    }
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  if (warp == C::CW) {
    // ============================================ factor producer ==========
    if (lane == 0) {
      // L2 prefetch cursor over this CTA's factor entries, PF entries ahead
      // of the loads, so that the loads into the ring hit L2.
      constexpr int PF = 12;
      int pf_ph = -1, pf_c = 0, pf_c1 = 0;
      auto pf_step = [&]() {
        while (pf_c >= pf_c1) {
          if (pf_ph >= p.nphase) return;
          if (++pf_ph >= p.nphase) return;
          const DfPhase& q = s_ph[pf_ph];
          if (q.type != DF_GEMV) { pf_c = pf_c1 = 0; continue; }
          share(q.T * q.nk, G, g, pf_c, pf_c1);
        }
        const DfPhase& q = s_ph[pf_ph];
        const int t = pf_c / q.nk, kc = pf_c - t * q.nk;
        const int kn = min(DF_KC, q.K - kc * DF_KC);
        prefetch_l2_bulk(p.pack + q.pack_off + (long long)t * q.K * 128 + (long long)kc * 32768,
                         (uint32_t)kn * 128u);
        ++pf_c;
      };
      for (int i = 0; i < PF; ++i) pf_step();
      int seq = 0;
      bool waited = false;
      for (int ph_i = 0; ph_i < p.nphase && !*abort_flag; ++ph_i) {
        const DfPhase& ph = s_ph[ph_i];
        int Ctot, c0, c1;
        if (ph.type == DF_ATTN) {
          if (!waited) { pdl_wait(); waited = true; }
          AttnSched s;
          attn_sched(p, s);
          Ctot = s.pre[8];
        } else {
          Ctot = ph.T * ph.nk;
        }
        if (Ctot == 0) continue;
        share(Ctot, G, g, c0, c1);
        for (int c = c0; c < c1; ++c, ++seq) {
          const int slot = seq % C::NSLOT;
          const uint32_t par = (uint32_t)(seq / C::NSLOT) & 1u;
          if (!tc::mbar_wait_sleep(empty + slot, par ^ 1u, abort_flag, p.status)) break;
          if (ph.type == DF_ATTN) {
            tc::mbar_arrive(full + slot);  // the K/V chunk comes from the other producer
          } else {
            const int t = c / ph.nk, kc = c - t * ph.nk;
            const uint32_t box = (uint32_t)min(DF_KC, ph.K - kc * DF_KC) * 64u;
            const uint8_t* e = p.pack + ph.pack_off + (long long)t * ph.K * 128 + (long long)kc * 32768;
            uint8_t* w = slots + slot * C::SLOT;
            mbar_arrive_expect(full + slot, 2u * box);
            bulk_g2s(w, e, box, full + slot);
            bulk_g2s(w + 16384, e + box, box, full + slot);
            pf_step();
          }
        }
      }
      if (*abort_flag) {
        const long long t0 = clock64();
        while (clock64() - t0 < 2000000) {}
      }
    }
  } else if (warp == C::CW + 1) {
    // ======================================== activation producer ==========
    if (lane == 0) {
      for (int i = 0; i < DF_NMAPS; ++i) tc::tma_prefetch_desc(&p.maps[i]);
      pdl_wait();
      int seq = 0;
      for (int ph_i = 0; ph_i < p.nphase && !*abort_flag; ++ph_i) {
        const DfPhase& ph = s_ph[ph_i];
        if (ph_i > 0) {
          // grid barrier: every CTA has finished stage ph_i - 1
          const long long t0 = clock64();
          while (ld_acquire(p.bar + ph_i - 1) < G) {
            if (*abort_flag) break;
            if (clock64() - t0 > tc::kWaitCycles) {
              *abort_flag = 1;
              atomicExch(p.status, DEV_STATUS_TIMEOUT);
              break;
            }
            __nanosleep(64);
          }
          if (*abort_flag) break;
        }
        int Ctot, c0, c1;
        AttnSched s;
        if (ph.type == DF_ATTN) {
          attn_sched(p, s);
          Ctot = s.pre[8];
        } else {
          Ctot = ph.T * ph.nk;
        }
        if (Ctot == 0) continue;
        share(Ctot, G, g, c0, c1);
        for (int c = c0; c < c1; ++c, ++seq) {
          const int slot = seq % C::NSLOT;
          const uint32_t par = (uint32_t)(seq / C::NSLOT) & 1u;
          if (!tc::mbar_wait_sleep(empty + slot, par ^ 1u, abort_flag, p.status)) break;
          uint8_t* base = slots + slot * C::SLOT;
          if (ph.type == DF_ATTN) {
            int b, h, kc;
            attn_entry(s, c, b, h, kc);
            const int NB = p.D >> 6;
            mbar_arrive_expect(full + slot, (uint32_t)(2 * NB * 8192));
            const int row = b * p.S_max + kc * 64;
            for (int bx = 0; bx < NB; ++bx) {
              tc::tma_load_2d(base + bx * 8192, &p.maps[0], full + slot, h * p.D + 64 * bx, row);
              tc::tma_load_2d(base + 16384 + bx * 8192, &p.maps[1], full + slot, h * p.D + 64 * bx, row);
            }
          } else {
            const int t = c / ph.nk, kc = c - t * ph.nk;
            const int k0 = kc * DF_KC;
            const int kn = min(DF_KC, ph.K - k0);
            int pi = 0;
            for (int i = 1; i < 3; ++i)
              if (i < ph.nprob && t >= ph.tile_start[i]) pi = i;
            const int esz = ph.a_f32 ? 4 : 2;
            const int nseg = ph.map == MAP_SWIGLU ? 2 : 1;
            const uint32_t rowbytes = (uint32_t)(kn * esz);
            mbar_arrive_expect(full + slot, rowbytes * (uint32_t)(nseg * p.B));
            uint8_t* a_s = base + C::W_BYTES;
            for (int sg = 0; sg < nseg; ++sg) {
              const int acol = (sg ? ph.a_col2 : ph.a_col[pi]) + k0;
              for (int m = 0; m < p.B; ++m) {
                const uint8_t* src = reinterpret_cast<const uint8_t*>(ph.a) +
                                     ((long long)m * ph.lda + acol) * esz;
                bulk_g2s(a_s + (sg * MT + m) * DF_KC * esz, src, rowbytes, full + slot);
              }
            }
          }
        }
      }
      if (*abort_flag) {
        const long long t0 = clock64();
        while (clock64() - t0 < 2000000) {}
      }
    }
  } else {
    // ================================================= consumers ==========
    pdl_wait();
    // lane bits: [1:0] 16-byte chunk, [2] row parity, [3] box, [..4] row lane;
    // a quarter warp then reads two consecutive 64-byte rows of one box.
    const int chunk = tid & 3, rsub = (tid >> 2) & 1, box = (tid >> 3) & 1, rowlane = tid >> 4;
    const int cg = box * 4 + chunk;
    const int row0 = 2 * rowlane + rsub;
    constexpr int RSTEP = C::CT / 8;
    int seq = 0;
    for (int ph_i = 0; ph_i < p.nphase; ++ph_i) {
      const DfPhase& ph = s_ph[ph_i];
      if (ph.type == DF_GEMV) {
        const int Ctot = ph.T * ph.nk;
        int c0, c1;
        share(Ctot, G, g, c0, c1);
        const int hi = box;
        float acc[MT][8];
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[m][j] = 0.f;
        int su = 0;
        const int t_first = c0 / (ph.nk > 0 ? ph.nk : 1);
        for (int c = c0; c < c1; ++c, ++seq) {
          const int slot = seq % C::NSLOT;
          const uint32_t par = (uint32_t)(seq / C::NSLOT) & 1u;
          tc::mbar_wait(full + slot, par, abort_flag, p.status);  // on abort: run on, results discarded
          const int t = c / ph.nk, kc = c - t * ph.nk;
          const int k0 = kc * DF_KC;
          const int kn = min(DF_KC, ph.K - k0);
          if (ph.pro == PRO_RMSNORM && c == c0) {
            // rstd of each row of x (the stage's input, complete after the barrier)
            const bf16* xb = reinterpret_cast<const bf16*>(ph.a);
            for (int m = 0; m < MT; ++m) {
              float ss = 0.f;
              if (m < p.B)
                for (int col = tid * 8; col < ph.K; col += C::CT * 8) {
                  const uint4 u = __ldcg(reinterpret_cast<const uint4*>(xb + (long long)m * ph.lda + col));
                  const float v[8] = {bf_lo(u.x), bf_hi(u.x), bf_lo(u.y), bf_hi(u.y),
                                      bf_lo(u.z), bf_hi(u.z), bf_lo(u.w), bf_hi(u.w)};
#pragma unroll
                  for (int j = 0; j < 8; ++j) ss = fmaf(v[j], v[j], ss);
                }
              ss = warp_sum(ss);
              if (lane == 0) red[warp * MT + m] = ss;
            }
            consumer_sync<C::CT>();
            if (tid < MT) {
              float ss = 0.f;
#pragma unroll
              for (int w = 0; w < C::CW; ++w) ss += red[w * MT + tid];
              s_rstd[tid] = rsqrtf(ss / (float)ph.K + p.eps);
            }
            consumer_sync<C::CT>();
          }
          const uint8_t* w = slots + slot * C::SLOT + hi * 16384 + (cg & 3) * 16;
          const uint8_t* a_s = slots + slot * C::SLOT + C::W_BYTES;
          if (ph.pro == PRO_RMSNORM)
            entry_mac<MT, 1, 0, RSTEP>(acc, w, a_s, 0, kn, row0, ph.norm_g + k0, s_rstd);
          else if (!ph.a_f32)
            entry_mac<MT, 0, 0, RSTEP>(acc, w, a_s, 0, kn, row0, nullptr, s_rstd);
          else
            entry_mac<MT, 0, 1, RSTEP>(acc, w, a_s, (ph.map == MAP_SWIGLU) ? hi : 0, kn, row0, nullptr,
                                       s_rstd);
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(empty + slot);

          const bool tile_end = (c == c1 - 1) || (kc == ph.nk - 1);
          if (!tile_end) continue;

          // ---- finish this CTA's part of tile t ----
#pragma unroll
          for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              float v = acc[m][j];
              v += __shfl_xor_sync(0xffffffffu, v, 4);
              v += __shfl_xor_sync(0xffffffffu, v, 16);
              acc[m][j] = 0.f;
              if ((lane & 20) == 0) red[(warp * MT + m) * 64 + cg * 8 + j] = v;
            }
          consumer_sync<C::CT>();
          constexpr int NOUT = MT * 64;
          const int e_first = t * ph.nk, e_last = min(Ctot - 1, t * ph.nk + ph.nk - 1);
          const int gf = owner_of(e_first, Ctot, G);
          const int gl = owner_of(e_last, Ctot, G);
          (void)gl;
          float* mypart = p.part + ((long long)g * DF_MAX_SU + (su < DF_MAX_SU ? su : DF_MAX_SU - 1)) *
                                       DF_PART_STRIDE;
          for (int o = tid; o < NOUT; o += C::CT) {
            float s = 0.f;
#pragma unroll
            for (int w8 = 0; w8 < C::CW; ++w8) s += red[(w8 * MT + (o >> 6)) * 64 + (o & 63)];
            if (gf == gl) scr[o] = s;
            else __stcg(mypart + o, s);
          }
          bool run_epi = true;
          if (gf != gl) {
            __threadfence();
            consumer_sync<C::CT>();
            if (tid == 0)
              *s_flag = (atomicAdd(p.tilecnt + t, 1) == count_owners(e_first, e_last, Ctot, G) - 1);
            consumer_sync<C::CT>();
            run_epi = *s_flag != 0;
            if (run_epi) {
              __threadfence();
              // SPL threads per output each sum a fixed stride of the
              // contributing CTAs; the SPL sums are added in fixed order.
              constexpr int SPL = C::CT / NOUT > 1 ? C::CT / NOUT : 1;
              const int o = tid % NOUT, sub = tid / NOUT;
              float sacc = 0.f;
              if (sub < SPL)
                for (int gg = gf + sub; gg <= gl; gg += SPL) {
                  if (Ctot < G && !share_nonempty(Ctot, G, gg)) continue;
                  const int c0g = gg * Ctot / G;
                  int sug = t - c0g / ph.nk;
                  sug = sug < DF_MAX_SU ? sug : DF_MAX_SU - 1;
                  sacc += __ldcg(p.part + ((long long)gg * DF_MAX_SU + sug) * DF_PART_STRIDE + o);
                }
              if (SPL > 1) {
                if (sub < SPL) red[sub * NOUT + o] = sacc;
                consumer_sync<C::CT>();
                if (tid < NOUT) {
                  float tot = 0.f;
#pragma unroll
                  for (int k2 = 0; k2 < SPL; ++k2) tot += red[k2 * NOUT + tid];
                  scr[tid] = tot;
                }
              } else {
                for (int o2 = tid; o2 < NOUT; o2 += C::CT) {
                  float tot = 0.f;
                  for (int gg = gf; gg <= gl; ++gg) {
                    if (Ctot < G && !share_nonempty(Ctot, G, gg)) continue;
                    const int c0g = gg * Ctot / G;
                    int sug = t - c0g / ph.nk;
                    sug = sug < DF_MAX_SU ? sug : DF_MAX_SU - 1;
                    tot += __ldcg(p.part + ((long long)gg * DF_MAX_SU + sug) * DF_PART_STRIDE + o2);
                  }
                  scr[o2] = tot;
                }
              }
              if (tid == 0) p.tilecnt[t] = 0;
            }
          }
          consumer_sync<C::CT>();
          if (run_epi) {
            int pi = 0;
            for (int i = 1; i < 3; ++i)
              if (i < ph.nprob && t >= ph.tile_start[i]) pi = i;
            const int tl = t - ph.tile_start[pi];
            const int Np = ph.N[pi];
            if (ph.epi == EPI_F32 || ph.epi == EPI_BF16) {
              for (int o = tid; o < NOUT; o += C::CT) {
                const int m = o >> 6, cc = o & 63;
                const int gc = out_col(ph, p.D, tl, cc);
                if (m >= p.B || gc >= Np) continue;
                float v = scr[o];
                if (ph.epi == EPI_F32) {
                  ph.out32[(long long)m * ph.ldo32 + ph.out_col[pi] + gc] = v;
                } else {
                  if (ph.resid) v += bf2f(__ldcg(ph.resid + (long long)m * ph.ldr + gc));
                  ph.out16[(long long)m * ph.ldo16 + gc] = f2bf(v);
                }
              }
            } else if (ph.epi == EPI_QKV) {
              const int half = p.D >> 1;
              const int kind = ph.kind[pi];
              for (int o = tid; o < MT * 32; o += C::CT) {
                const int m = o >> 5, cc = o & 31;
                if (m >= p.B) continue;
                int pos = p.seqlens[m];
                pos = pos < 0 ? 0 : (pos >= p.S_max ? p.S_max - 1 : pos);
                const int glo = out_col(ph, p.D, tl, cc);
                const int i = glo % p.D;
                float lo = scr[m * 64 + cc], hv = scr[m * 64 + cc + 32];
                if (kind < 2) {
                  const float cs = p.rope_cos[(long long)pos * half + i];
                  const float sn = p.rope_sin[(long long)pos * half + i];
                  const float l2 = lo * cs - hv * sn;
                  hv = hv * cs + lo * sn;
                  lo = l2;
                }
                bf16* dst;
                if (kind == 0) dst = ph.out16 + (long long)m * ph.ldo16;
                else dst = (kind == 1 ? p.k_cache : p.v_cache) + ((long long)m * p.S_max + pos) * (p.H * p.D);
                dst[glo] = f2bf(lo);
                dst[glo + half] = f2bf(hv);
              }
            } else {  // EPI_SWIGLU
              for (int o = tid; o < MT * 32; o += C::CT) {
                const int m = o >> 5, cc = o & 31;
                const int fc = 32 * tl + cc;
                if (m >= p.B || fc >= Np) continue;
                const float gv = scr[m * 64 + cc], uv = scr[m * 64 + cc + 32];
                ph.out16[(long long)m * ph.ldo16 + fc] = f2bf(gv / (1.f + expf(-gv)) * uv);
              }
            }
          }
          consumer_sync<C::CT>();
          ++su;
          (void)t_first;
        }
      } else {
        // ---------------------------------------------- attention stage --
        // Each consumer warp owns 64 / CW keys of every 64-key entry and keeps
        // its own online-softmax state (m, l, o) over all entries of a
        // (batch, head) pair; lanes own D / 32 dimensions.  Warps merge once
        // per pair, then CTAs merge through the partial slots.
        AttnSched s;
        attn_sched(p, s);
        const int Ctot = s.pre[8];
        int c0, c1;
        share(Ctot, G, g, c0, c1);
        const int D = p.D;
        const int EPL = D >> 5;               // 4 (D = 128) or 2 (D = 64)
        constexpr int KPW = 64 / C::CW;       // keys per warp per entry
        float* wm = scr;                      // [CW]      warp m
        float* wl = scr + 32;                 // [CW]      warp l
        float* wo = scr + 64;                 // [CW][128] warp o
        float qv[4] = {0.f, 0.f, 0.f, 0.f};
        float m_w = -INFINITY, l_w = 0.f;
        float ov[4] = {0.f, 0.f, 0.f, 0.f};
        int su = 0;
        for (int c = c0; c < c1; ++c, ++seq) {
          int b, h, kc;
          attn_entry(s, c, b, h, kc);
          const int pair_first = s.pre[b] + h * s.nk[b];
          const int pair_last = pair_first + s.nk[b] - 1;
          const int slot = seq % C::NSLOT;
          const uint32_t par = (uint32_t)(seq / C::NSLOT) & 1u;
          tc::mbar_wait(full + slot, par, abort_flag, p.status);  // on abort: run on, results discarded
          if (c == c0 || kc == 0) {
            m_w = -INFINITY; l_w = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) ov[e] = 0.f;
            const bf16* qp = p.q + ((long long)b * p.H + h) * D + lane * EPL;
#pragma unroll
            for (int e = 0; e < 4; ++e) qv[e] = e < EPL ? bf2f(__ldcg(qp + e)) * p.scale_log2 : 0.f;
          }
          const uint8_t* kb = slots + slot * C::SLOT;
          const uint8_t* vb = kb + 16384;
          // this lane's dims: d0 = lane * EPL .. + EPL (one 8- or 4-byte piece)
          const int d0 = lane * EPL;
          const int bx = d0 >> 6, ch = (d0 & 63) >> 3, sub = (d0 & 7) * 2;
          float sc4[KPW];
#pragma unroll
          for (int i = 0; i < KPW; ++i) {
            const int j = warp * KPW + i;
            const uint8_t* kp = kb + bx * 8192 + j * 128 + ((ch ^ (j & 7)) << 4) + sub;
            float dot = 0.f;
            if (EPL == 4) {
              const uint2 u = *reinterpret_cast<const uint2*>(kp);
              dot = qv[0] * bf_lo(u.x) + qv[1] * bf_hi(u.x) + qv[2] * bf_lo(u.y) + qv[3] * bf_hi(u.y);
            } else {
              const uint32_t u = *reinterpret_cast<const uint32_t*>(kp);
              dot = qv[0] * bf_lo(u) + qv[1] * bf_hi(u);
            }
            sc4[i] = dot;
          }
#pragma unroll
          for (int i = 0; i < KPW; ++i) {
            sc4[i] = warp_sum(sc4[i]);
            const int key = kc * 64 + warp * KPW + i;
            if (key >= s.L[b]) sc4[i] = -INFINITY;
          }
          float mb = sc4[0];
#pragma unroll
          for (int i = 1; i < KPW; ++i) mb = fmaxf(mb, sc4[i]);
          const float mn = fmaxf(m_w, mb);
          if (mn != -INFINITY) {
            const float corr = (m_w == -INFINITY) ? 0.f : exp2f(m_w - mn);
            l_w *= corr;
#pragma unroll
            for (int e = 0; e < 4; ++e) ov[e] *= corr;
#pragma unroll
            for (int i = 0; i < KPW; ++i) {
              const float pj = (sc4[i] == -INFINITY) ? 0.f : exp2f(sc4[i] - mn);
              l_w += pj;
              const int j = warp * KPW + i;
              const uint8_t* vp = vb + bx * 8192 + j * 128 + ((ch ^ (j & 7)) << 4) + sub;
              if (EPL == 4) {
                const uint2 u = *reinterpret_cast<const uint2*>(vp);
                ov[0] = fmaf(pj, bf_lo(u.x), ov[0]); ov[1] = fmaf(pj, bf_hi(u.x), ov[1]);
                ov[2] = fmaf(pj, bf_lo(u.y), ov[2]); ov[3] = fmaf(pj, bf_hi(u.y), ov[3]);
              } else {
                const uint32_t u = *reinterpret_cast<const uint32_t*>(vp);
                ov[0] = fmaf(pj, bf_lo(u), ov[0]); ov[1] = fmaf(pj, bf_hi(u), ov[1]);
              }
            }
            m_w = mn;
          }
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(empty + slot);

          const bool pair_end = (c == c1 - 1) || (c == pair_last);
          if (!pair_end) continue;
          // ---- merge the warps of this CTA for pair (b, h) ----
          if (lane == 0) { wm[warp] = m_w; wl[warp] = l_w; }
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (e < EPL) wo[warp * 128 + lane * EPL + e] = ov[e];
          consumer_sync<C::CT>();
          float Mc = -INFINITY;
#pragma unroll
          for (int w2 = 0; w2 < C::CW; ++w2) Mc = fmaxf(Mc, wm[w2]);
          float Lc = 0.f, oc = 0.f;
#pragma unroll
          for (int w2 = 0; w2 < C::CW; ++w2) {
            const float wgt = (wm[w2] == -INFINITY) ? 0.f : exp2f(wm[w2] - Mc);
            Lc += wgt * wl[w2];
            if (tid < D) oc += wgt * wo[w2 * 128 + tid];
          }
          const int pair = b * p.H + h;
          const int gf = owner_of(pair_first, Ctot, G), gl = owner_of(pair_last, Ctot, G);
          float* mypart = p.part + ((long long)g * DF_MAX_SU + (su < DF_MAX_SU ? su : DF_MAX_SU - 1)) *
                                       DF_PART_STRIDE;
          if (gf == gl) {
            if (tid < D) p.att[((long long)b * p.H + h) * D + tid] = f2bf(oc / Lc);
          } else {
            if (tid < D) __stcg(mypart + 2 + tid, oc);
            if (tid == 0) { __stcg(mypart, Mc); __stcg(mypart + 1, Lc); }
            __threadfence();
            consumer_sync<C::CT>();
            if (tid == 0)
              *s_flag = (atomicAdd(p.tilecnt + pair, 1) == count_owners(pair_first, pair_last, Ctot, G) - 1);
            consumer_sync<C::CT>();
            if (*s_flag) {
              __threadfence();
              float* cm = scr + 64 + C::CW * 128;   // [32] contributor m
              float* cl = cm + 32;                   // [32] contributor l
              int* cs = reinterpret_cast<int*>(cl + 32);  // [33] slot index, count
              if (tid == 0) {
                int n = 0;
                for (int gg = gf; gg <= gl && n < 32; ++gg) {
                  if (Ctot < G && !share_nonempty(Ctot, G, gg)) continue;
                  const int c0g = gg * Ctot / G;
                  int b2, h2, k2;
                  attn_entry(s, c0g, b2, h2, k2);
                  int sug = pair - (b2 * p.H + h2);
                  sug = sug < DF_MAX_SU ? sug : DF_MAX_SU - 1;
                  cs[n++] = gg * DF_MAX_SU + sug;
                }
                cs[32] = n;
              }
              consumer_sync<C::CT>();
              const int ncon = cs[32];
              if (tid < ncon) {
                const float* pp = p.part + (long long)cs[tid] * DF_PART_STRIDE;
                cm[tid] = __ldcg(pp);
                cl[tid] = __ldcg(pp + 1);
              }
              consumer_sync<C::CT>();
              float Mg = -INFINITY;
              for (int k2 = 0; k2 < ncon; ++k2) Mg = fmaxf(Mg, cm[k2]);
              float Lg = 0.f;
              for (int k2 = 0; k2 < ncon; ++k2)
                Lg += (cm[k2] == -INFINITY) ? 0.f : exp2f(cm[k2] - Mg) * cl[k2];
              float* oh = scr + 64;  // reuse the warp-o area: [CT / D][D]
              {
                const int KG2 = C::CT / D;
                const int dd = tid % D, kg = tid / D;
                float oo = 0.f;
                for (int k2 = kg; k2 < ncon; k2 += KG2) {
                  const float wgt = (cm[k2] == -INFINITY) ? 0.f : exp2f(cm[k2] - Mg);
                  oo += wgt * __ldcg(p.part + (long long)cs[k2] * DF_PART_STRIDE + 2 + dd);
                }
                oh[kg * D + dd] = oo;
              }
              consumer_sync<C::CT>();
              if (tid < D) {
                float o = 0.f;
                for (int k2 = 0; k2 < C::CT / D; ++k2) o += oh[k2 * D + tid];
                p.att[((long long)b * p.H + h) * D + tid] = f2bf(o / Lg);
              }
              if (tid == 0) p.tilecnt[pair] = 0;
            }
          }
          consumer_sync<C::CT>();
          ++su;
        }
      }
      // ---- this CTA is done with stage ph_i ----
      // Stores of this stage must be visible to the next stage's TMA / bulk
      // copies (async proxy) issued by other CTAs.
      asm volatile("fence.proxy.async.global;" ::: "memory");
      consumer_sync<C::CT>();
      if (tid == 0) {
        __threadfence();
        red_release_add(p.bar + ph_i, 1);
      }
    }
  }

  __syncthreads();
  if (tid == 0) {
    // The last CTA to finish resets the stage counters for the next launch.
    __threadfence();
    if (atomicAdd(p.done, 1) == G - 1) {
      for (int i = 0; i < DF_NPHASE; ++i) p.bar[i] = 0;
      __threadfence();
      *p.done = 0;
    }
  }
}

// ------------------------------------------------------------ the pack --
// Entry (t, kc) of a stage -- rows [256 kc, 256 kc + kn) of column tile t --
// is stored as box 0 then box 1, each [kn x 32] bf16 row-major (64-byte
// rows), at byte offset  stage_off + t * K * 128 + kc * 32768.  A box's 32
// source columns (and, for the SwiGLU map, source rows) follow the stage's
// output map; columns at or beyond the factor's width are zero.
struct PackStage {
  long long off;
  int K, T, map, nprob, w_row2;
  int tile_start[4];
  int N[3];
  const bf16* src[3];
  long long ld[3];
};
struct PackParams {
  PackStage st[DF_NPHASE];
  int nstage, D;
  long long total;
  uint8_t* dst;
};

__global__ void __launch_bounds__(256) decode_pack_kernel(const __grid_constant__ PackParams p) {
  const long long n16 = p.total >> 4;
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < n16;
       q += (long long)gridDim.x * blockDim.x) {
    const long long byte = q << 4;
    int i = 0;
    while (i + 1 < p.nstage && byte >= p.st[i + 1].off) ++i;
    const PackStage& st = p.st[i];
    long long rem = byte - st.off;
    const long long tile_bytes = (long long)st.K * 128;
    const int t = (int)(rem / tile_bytes);
    rem -= (long long)t * tile_bytes;
    const int kc = (int)(rem >> 15);
    rem -= (long long)kc << 15;
    const int k0 = kc * DF_KC;
    const int kn = min(DF_KC, st.K - k0);
    const int box = rem >= (long long)kn * 64 ? 1 : 0;
    rem -= (long long)box * kn * 64;
    const int row = (int)(rem >> 6), chunk = (int)((rem >> 4) & 3);
    int pi = 0;
    for (int j = 1; j < 3; ++j)
      if (j < st.nprob && t >= st.tile_start[j]) pi = j;
    const int tl = t - st.tile_start[pi];
    long long srow = k0 + row;
    int col;
    if (st.map == MAP_PLAIN) {
      col = 64 * tl + 32 * box;
    } else if (st.map == MAP_ROPE) {
      const int tph = p.D >> 6, hh = tl / tph, j = tl - hh * tph;
      col = hh * p.D + 32 * j + box * (p.D >> 1);
    } else {
      col = 32 * tl;
      srow += box * st.w_row2;
    }
    col += 8 * chunk;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (col < st.N[pi]) v = __ldg(reinterpret_cast<const uint4*>(st.src[pi] + srow * st.ld[pi] + col));
    *reinterpret_cast<uint4*>(p.dst + byte) = v;
  }
}

}  // namespace

// ------------------------------------------------------------------ host --

int decode_fused_supported(int B, int d, int D, int r, int r_f) {
  return B >= 1 && B <= 8 && (D == 64 || D == 128) && d % 64 == 0 && r % 8 == 0 && r_f % 8 == 0;
}

// Stage table of one fused decode layer.  Activation pointers may be null
// (when only the pack layout is wanted); Q, if given, receives each stage's
// factor sources for the pack kernel.  Returns the pack size in bytes.
long long build_stages(const DecodeLayerDesc& L, bf16* x, bf16* qbuf, const bf16* att, bf16* hbuf,
                       float* z, DfPhase* P, PackStage* Q) {
  const int d = L.d, r = L.r, rf = L.r_f, f = L.f;
  memset(P, 0, sizeof(DfPhase) * DF_NPHASE);
  long long off = 0;
  auto gemv = [&](int i, int pro, int epi, int map, int K, const bf16* const* src, const long long* ld) {
    DfPhase& ph = P[i];
    ph.type = DF_GEMV; ph.pro = pro; ph.epi = epi; ph.map = map; ph.K = K;
    ph.nk = ceil_div(K, DF_KC);
    int T = 0;
    for (int j = 0; j < ph.nprob; ++j) {
      ph.tile_start[j] = T;
      T += (map == MAP_SWIGLU) ? ceil_div(ph.N[j], 32) : ceil_div(ph.N[j], 64);
    }
    for (int j = ph.nprob; j < 4; ++j) ph.tile_start[j] = T;
    ph.T = T;
    ph.pack_off = off;
    if (Q) {
      PackStage& q = Q[i];
      q.off = off; q.K = K; q.T = T; q.map = map; q.nprob = ph.nprob; q.w_row2 = ph.w_row2;
      for (int j = 0; j < 4; ++j) q.tile_start[j] = ph.tile_start[j];
      for (int j = 0; j < ph.nprob; ++j) { q.N[j] = ph.N[j]; q.src[j] = src[j]; q.ld[j] = ld[j]; }
    }
    off += (long long)T * K * 128;
  };
  // 0: z_qkv = rmsnorm(x) . [U_q | U_k | U_v]
  P[0].nprob = 3;
  for (int i = 0; i < 3; ++i) { P[0].N[i] = r; P[0].out_col[i] = i * r; }
  P[0].a = x; P[0].a_f32 = 0; P[0].lda = d; P[0].norm_g = L.g1;
  P[0].out32 = z; P[0].ldo32 = 3 * r;
  { const long long ld[3] = {r, r, r}; gemv(0, PRO_RMSNORM, EPI_F32, MAP_PLAIN, d, L.U, ld); }
  // 1: q, k, v = z . V  (+ RoPE; k, v appended at cache_seqlens)
  P[1].nprob = 3;
  for (int i = 0; i < 3; ++i) { P[1].N[i] = d; P[1].a_col[i] = i * r; P[1].kind[i] = i; }
  P[1].a = z; P[1].a_f32 = 1; P[1].lda = 3 * r;
  P[1].out16 = qbuf; P[1].ldo16 = d;
  { const long long ld[3] = {d, d, d}; gemv(1, PRO_F32, EPI_QKV, MAP_ROPE, r, L.V, ld); }
  // 2: attention
  P[2].type = DF_ATTN;
  // 3: z = att . U_o
  P[3].nprob = 1; P[3].N[0] = r;
  P[3].a = att; P[3].a_f32 = 0; P[3].lda = d; P[3].out32 = z; P[3].ldo32 = r;
  { const long long ld[1] = {r}; gemv(3, PRO_BF16, EPI_F32, MAP_PLAIN, d, &L.U_o, ld); }
  // 4: x += z . V_o
  P[4].nprob = 1; P[4].N[0] = d;
  P[4].a = z; P[4].a_f32 = 1; P[4].lda = r; P[4].out16 = x; P[4].ldo16 = d; P[4].resid = x; P[4].ldr = d;
  { const long long ld[1] = {d}; gemv(4, PRO_F32, EPI_BF16, MAP_PLAIN, r, &L.V_o, ld); }
  // 5: z = rmsnorm(x) . U_gu
  P[5].nprob = 1; P[5].N[0] = 2 * rf;
  P[5].a = x; P[5].a_f32 = 0; P[5].lda = d; P[5].norm_g = L.g2; P[5].out32 = z; P[5].ldo32 = 2 * rf;
  { const long long ld[1] = {2 * rf}; gemv(5, PRO_RMSNORM, EPI_F32, MAP_PLAIN, d, &L.U_gu, ld); }
  // 6: h = SiLU(z_g V_g) * (z_u V_u)
  P[6].nprob = 1; P[6].N[0] = f; P[6].a_col[0] = 0; P[6].a_col2 = rf; P[6].w_row2 = rf;
  P[6].a = z; P[6].a_f32 = 1; P[6].lda = 2 * rf; P[6].out16 = hbuf; P[6].ldo16 = f;
  { const long long ld[1] = {f}; gemv(6, PRO_F32, EPI_SWIGLU, MAP_SWIGLU, rf, &L.V_gu, ld); }
  // 7: z = h . U_dn
  P[7].nprob = 1; P[7].N[0] = rf;
  P[7].a = hbuf; P[7].a_f32 = 0; P[7].lda = f; P[7].out32 = z; P[7].ldo32 = rf;
  { const long long ld[1] = {rf}; gemv(7, PRO_BF16, EPI_F32, MAP_PLAIN, f, &L.U_dn, ld); }
  // 8: x += z . V_dn
  P[8].nprob = 1; P[8].N[0] = d;
  P[8].a = z; P[8].a_f32 = 1; P[8].lda = rf; P[8].out16 = x; P[8].ldo16 = d; P[8].resid = x; P[8].ldr = d;
  { const long long ld[1] = {d}; gemv(8, PRO_F32, EPI_BF16, MAP_PLAIN, rf, &L.V_dn, ld); }
  return off;
}

long long decode_pack_bytes(const DecodeLayerDesc& L) {
  DfPhase P[DF_NPHASE];
  return build_stages(L, nullptr, nullptr, nullptr, nullptr, nullptr, P, nullptr);
}

int decode_pack_launch(const DecodeLayerDesc& L, void* dst, long long bytes, int sm_count,
                       cudaStream_t stream) {
  DfPhase P[DF_NPHASE];
  PackParams pp;
  memset(&pp, 0, sizeof(pp));
  const long long need = build_stages(L, nullptr, nullptr, nullptr, nullptr, nullptr, P, pp.st);
  if (bytes < need) return FLASHSVD_ERR_INVALID_ARG;
  // Stage 2 (attention) holds no factors: an empty range at stage 3's
  // offset lets the pack kernel's stage search pass over it.
  pp.st[2] = pp.st[3];
  pp.st[2].T = 0;
  pp.nstage = DF_NPHASE;
  pp.D = L.D;
  pp.total = need;
  pp.dst = static_cast<uint8_t*>(dst);
  const long long n16 = need >> 4;
  const int grid = (int)std::min<long long>((n16 + 255) / 256, (long long)sm_count * 8);
  decode_pack_kernel<<<grid, 256, 0, stream>>>(pp);
  return cuda_status(cudaGetLastError());
}

int decode_fused_launch(const DecodeLayerDesc& L, bf16* x, bf16* kc, bf16* vc, const int* seqlens,
                        int B, int S_max, bf16* qbuf, bf16* att, bf16* hbuf, float* z, float* part,
                        int* tilecnt, int* bar, int* done, int* status, int sm_count,
                        cudaStream_t stream) {
  if (!L.pack) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  DfParams p;
  memset(&p, 0, sizeof(p));
  DfPhase* P = p.ph;
  const long long pack_bytes = build_stages(L, x, qbuf, att, hbuf, z, P, nullptr);
  p.pack = static_cast<const uint8_t*>(L.pack);
  const long long HD = (long long)L.H * L.D;
  FSVD_TRY(encode_map(&p.maps[0], kc, (long long)B * S_max, HD, HD, 64, 64, true));
  FSVD_TRY(encode_map(&p.maps[1], vc, (long long)B * S_max, HD, HD, 64, 64, true));
  p.nphase = 9;

  // Every CTA's share of a stage may touch at most DF_MAX_SU tiles.
  const int G = sm_count;
  for (int i = 0; i < 9; ++i) {
    if (P[i].type != DF_GEMV) continue;
    const int Ctot = P[i].T * P[i].nk;
    const int per = ceil_div(Ctot, G);
    if (ceil_div(per, P[i].nk) + 1 > DF_MAX_SU || P[i].T > 4096) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  }
  // attention: a CTA's share spans at most (B*H)/G + 2 (batch, head) pairs
  if ((B * L.H) / G + 3 > DF_MAX_SU || B * L.H > 4096) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;

  p.B = B; p.H = L.H; p.D = L.D; p.S_max = S_max;
  p.eps = L.eps;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)L.D);
  p.seqlens = seqlens; p.k_cache = kc; p.v_cache = vc;
  p.rope_cos = L.rope_cos; p.rope_sin = L.rope_sin;
  p.q = qbuf; p.att = att;
  p.part = part; p.tilecnt = tilecnt; p.bar = bar; p.done = done; p.status = status;

  const double bytes = (double)pack_bytes + 2.0 * 2.0 * B * (double)S_max * HD;
  const LaunchTag tag{"decode_layer_fused", bytes, 0.0};

#define FSVD_DF_LAUNCH(MT_)                                                                          \
  {                                                                                                  \
    auto kern = decode_layer_kernel<MT_>;                                                            \
    static bool configured = false;                                                                  \
    if (!configured) {                                                                               \
      FSVD_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, DfCfg<MT_>::SMEM)); \
      configured = true;                                                                             \
    }                                                                                                \
    return launch_pdl(tag, kern, dim3(G), dim3(DfCfg<MT_>::THREADS), (size_t)DfCfg<MT_>::SMEM, stream, p);   \
  }
  if (B <= 1) FSVD_DF_LAUNCH(1)
  if (B <= 2) FSVD_DF_LAUNCH(2)
  if (B <= 4) FSVD_DF_LAUNCH(4)
  FSVD_DF_LAUNCH(8)
#undef FSVD_DF_LAUNCH
}

}  // namespace fsvd
