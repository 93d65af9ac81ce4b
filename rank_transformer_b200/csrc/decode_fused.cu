// Fused decode layer: the whole decode step of one low-rank decoder layer in
// one persistent kernel (one CTA per SM).
//
// FlashSVD v1.5 (gist.science explainer), Technical Summary: decode is
// memory-bound (Problem Statement), the present token's q/k/v are rebuilt
// through the low-rank projections and the history is read from a dense KV
// cache (Methodology 2), gate and up share one packed projection
// (Methodology 3), and the per-layer decode body is one replay unit
// (Methodology 4).  Here that replay unit is a single kernel with nine
// stages separated by grid barriers:
//   0  z = rmsnorm(x) [U_q | U_k | U_v]      5  z = rmsnorm(x') U_gu
//   1  q, k, v = z V (+RoPE)                 6  h = SiLU(z_g V_g) (z_u V_u)
//   2  attention over the dense cache        7  z = h U_dn
//   3  z = a U_o                             8  x'' = x' + z V_dn
//   4  x' = x + z V_o
// followed by a short final pass that writes x'' back over x.
//
// Factors.  They are read from the layer's decode pack: every factor matrix
// re-tiled once, at load time, so that each ring entry (256 rows x 64 output
// columns, laid out as 16 per-warp regions of 4 columns) is one contiguous
// block of HBM, stored in consumption order.  Whole blocks stream near the
// HBM copy rate; 64- or 128-byte row pieces spaced at the matrix pitch do
// not.
//
// Reduction ("reduce on read").  A CTA's share of a stage is a contiguous
// range of (tile, 256-row chunk) entries, so a column tile's K range is
// split over a few CTAs.  Consumer warp w owns columns 4w..4w+3 of every
// entry, so a tile's column sums are complete inside each warp; the CTA
// writes one fp32 partial per tile it touched and nothing else: no atomics,
// no last-arriver combine.  After the grid
// barrier, each CTA builds the stage input it needs by summing those
// partials (in CTA order, so every reader gets the same bits) and applying
// the previous stage's epilogue as it reads: RoPE and bf16 rounding of q/k/v,
// residual add and RMSNorm, SwiGLU, and the softmax merge of attention
// partials.  The new key and value enter attention from these sums; the CTA
// that owns a sequence's last cache chunk also appends them to the cache.
// Hence the K/V chunks themselves depend on no stage and are loaded as soon
// as ring slots free up.
//
// Roles per CTA (CW consumer warps + 1 producer warp):
//   warp CW   producer: fills every ring entry in order -- one bulk copy
//             per pack entry for the GEMV stages (prefetched two entries
//             ahead into L2), TMA loads of 64-key cache chunks for attention;
//             it never waits for activations.
//   consumers multiply-accumulate ring entries against the stage input
//             built in shared memory, and run attention with per-warp
//             online-softmax state.  The next GEMV stage's schedule record
//             and the next layer's stage table are copied (cp.async) into
//             second shared-memory buffers while the current stage runs.
// All waits are bounded; a timeout sets the device status word.
#include <algorithm>
#include <cstring>
#include <vector>

#include "kernels.h"
#include "tc.cuh"

namespace fsvd {

namespace {

constexpr int DF_KC = 256;            // rows per ring entry
constexpr int DF_MAX_SU = 16;         // tiles (or attention pairs) per CTA and stage
constexpr int DF_PART_STRIDE = 640;   // floats per partial slot (>= 4 x 64, >= 4 + 128)
constexpr int DF_NPHASE = 9;
constexpr int DF_ABUF_COLS = 4096;    // floats per row of the stage-input buffer at MT = 1
constexpr int DF_ABUF_WIDE = 5120;    // ... at MT >= 2 (a SwiGLU stage of r_f up to 2560)
// Stage-input row width of the MT-row kernel (the MT = 1 kernel has no
// shared memory left beside its six-slot ring for the wider buffer).
__host__ __device__ constexpr int df_acols(int MT) { return MT == 1 ? DF_ABUF_COLS : DF_ABUF_WIDE; }
constexpr int DF_MAX_PAIRS = 8;       // attention (batch, head) pairs per CTA
constexpr int DF_MAX_NK = 64;         // 256-row chunks per factor (K <= 16384)
constexpr int DF_CMAX = 15;           // contributing CTAs per tile (or pair) read
constexpr int DF_MAX_UNITS = 96;      // tiles (or pairs) read per stage and CTA

#ifdef FLASHSVD_TRACE
// Stage timeline (trace builds only; the product build compiles none of
// it): per (layer, stage, CTA) of the last launch, four points -- stage
// entry, previous stage complete on every CTA (grid barrier passed), stage
// input built, stage done (before the release) -- each as %globaltimer ns
// (comparable across SMs) and clock64 cycles (exact within a CTA).
constexpr int DF_TRACE_LAYERS = 64;
constexpr int DF_TRACE_CTAS = 148;
__device__ unsigned long long g_df_trace[DF_TRACE_LAYERS][9][DF_TRACE_CTAS][2][4];
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
#define DF_TRACE(l, ph, k)                                                     \
  do {                                                                         \
    if (tid == 0 && (l) < DF_TRACE_LAYERS && g < DF_TRACE_CTAS) {              \
      g_df_trace[l][ph][g][0][k] = global_ns();                                \
      g_df_trace[l][ph][g][1][k] = (unsigned long long)clock64();              \
    }                                                                          \
  } while (0)
#else
#define DF_TRACE(l, ph, k) \
  do {                     \
  } while (0)
#endif

enum { DF_GEMV = 0, DF_ATTN = 1 };
// How a stage's input is built from what the previous stage left.
// SRC_XOUT (stage 0 of every layer after the first): the previous layer's
// output x'' = x' + z V_dn, summed from its last stage's partials.
enum { SRC_X = 0, SRC_PART = 1, SRC_ATT = 2, SRC_XMID = 3, SRC_SWIGLU = 4, SRC_XOUT = 5 };

struct DfPhase {
  int type, map, src, norm;
  int nprob;
  int tile_start[4];
  int T, K, nk;
  int N[3];
  int a_col2;          // SwiGLU stage: offset of the up half in the previous output
  long long pack_off;  // byte offset of this stage's entries from the layer's pack
                       // (a shared factor's entries live in an earlier layer's pack)
  const bf16* norm_g;
  int shared;          // entries read by several layers: loaded with an L2 evict-last hint
  int ustride;         // SRC_PART stages: unit-table slots per (input chunk, segment)
  int pad_[2];
};

// A 256-row input chunk of a SRC_PART stage spans 4 previous-stage column
// tiles of 64 when it starts on a tile boundary (always for one segment;
// for the SwiGLU stage's second segment when the up half's offset r_f is a
// multiple of 64), else 5.
inline int part_ustride(const DfPhase& ph) {
  return (ph.map == MAP_SWIGLU && ph.a_col2 % 64) ? 5 : 4;
}

// Per (stage, CTA) schedule record, built on the host with the pack: the
// input chunks (problem << 8 | 256-row chunk) of the CTA's entries in
// first-use order, the chunk of each entry, and the contributor table of the
// previous-stage tiles those chunks draw on.  Records 0..8 follow the
// stages (attention-dependent tables are filled on the device); record 9
// serves the final pass (tiles g, g + G, ... of the last stage) and record 10
// the next layer's first stage (every tile of the last stage).
constexpr int DF_NREC = DF_NPHASE + 2;
constexpr int DF_MAX_E = 48;  // entries per CTA and stage
struct SchedRec {
  int n, nunits, pad0, pad1;
  int clist[16];
  uint8_t chunk_of[DF_MAX_E];
  short utab[DF_MAX_UNITS][16];
};
static_assert(sizeof(SchedRec) % 128 == 0, "schedule records stay 128-byte aligned");

// One decoder layer as the kernel sees it.
struct alignas(64) DfLayer {
  CUtensorMap kmap, vmap;      // the K and V cache views [B * S_max x H * D]
  const uint8_t* pack;
  const SchedRec* sched;       // [DF_NREC][G], inside the pack
  bf16* k_cache;
  bf16* v_cache;
  DfPhase ph[DF_NPHASE];
};

struct DfParams {
  DfLayer inl;              // the layer, when layers is null
  const DfLayer* layers;    // [nlayer] in device memory (several layers per launch)
  int nlayer;
  int B, H, D, S_max, d;
  float eps, scale_log2;
  const int* seqlens;
  bf16* x;        // input of the first layer; output of the last
  bf16* xm;       // x' (after a layer's attention block) [B x d]
  const float* rope_cos;
  const float* rope_sin;
  float* part;    // [2][G][DF_MAX_SU][DF_PART_STRIDE]: global stage gs writes half gs & 1
  int* bar;       // [DF_NPHASE] arrivals per stage, accumulated over the layers
  int* done;
  int* status;
  int drop_arrival;  // test hook: CTA 0 does not arrive at the first grid barrier
};

template <int MT>
struct DfCfg {
  static constexpr int CW = 16;                      // consumer warps
  static constexpr int CT = CW * 32;                 // consumer threads
  static constexpr int THREADS = CT + 32;            // + the producer warp
  static constexpr int SLOT = 32768;
  static constexpr int NSLOT = MT == 1 ? 6 : (MT == 2 ? 5 : 4);
  static constexpr int ACOLS = df_acols(MT);
  static constexpr int ABUF_BYTES = MT * ACOLS * 4;
  static constexpr int RED_BYTES = 512;              // per-warp sums of squares (RMSNorm)
  static constexpr int SCR_BYTES = (64 + CW * 128) * 4;
  static constexpr int MISC_BYTES = 6656;  // two schedule records, rstd, attention schedule
  static constexpr int BAR_BYTES = 512;
  static constexpr int PH_BYTES = 2 * 896;  // two copies of a layer's record tail (stage table)
  static constexpr int SMEM = 1024 + NSLOT * SLOT + ABUF_BYTES + RED_BYTES + SCR_BYTES + MISC_BYTES +
                              BAR_BYTES + PH_BYTES;
  static_assert(SMEM <= 232448, "shared memory budget");
};

template <int N>
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void prefetch_l2_bulk(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// Bulk copies and L2 prefetches with an L2 cache policy (evict-last for
// factors that several layers read: shared bases).
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void prefetch_l2_bulk_hint(const void* src, uint32_t bytes, uint64_t pol) {
  asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], %1, %2;" ::"l"(src), "r"(bytes), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          tc::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(tc::smem_u32(bar)), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          tc::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ float bf_round(float v) { return bf2f(f2bf(v)); }
// 2^x with the hardware approximation (relative error ~2^-22; 2^-inf = +0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Bounded wait until stage counter *bar reaches target.
__device__ __forceinline__ void grid_wait(const int* bar, int target, volatile int* abort_flag, int* status) {
  const long long t0 = clock64();
  while (ld_acquire(bar) < target) {
    if (*abort_flag) return;
    if (clock64() - t0 > tc::kWaitCycles) {
      *abort_flag = 1;
      atomicExch(status, DEV_STATUS_TIMEOUT);
      return;
    }
    __nanosleep(32);
  }
}

// Contiguous share [c0, c1) of C entries for CTA g of G; owner of entry c.
// (32-bit: C * G stays below 2^31 for every stage the host accepts.)
__device__ __forceinline__ void share(int C, int G, int g, int& c0, int& c1) {
  c0 = g * C / G;
  c1 = (g + 1) * C / G;
}
__host__ __device__ __forceinline__ int owner_of(int c, int C, int G) { return ((c + 1) * G - 1) / C; }
__host__ __device__ __forceinline__ bool share_nonempty(int C, int G, int g) {
  return (g + 1) * C / G > g * C / G;
}

// Attention entry layout: for each batch row b, H heads x ne_b entries of
// 64 keys, ne_b = max(nk_b, m) with nk_b the chunks of the current length
// L_b = position + 1; entries past nk_b are empty (nothing loaded or
// computed).  The entries are split evenly over the first Ga CTAs.  Two
// per-CTA limits follow from the choice of Ga and m, whatever the lengths:
//  - a pair's entries (at most Ctot / H of them) span at most
//    ceil(Ga / H) + 1 <= DF_CMAX CTAs, as Ga <= (DF_CMAX - 1) H;
//  - a share of S <= ceil(Ctot / Ga) entries meets at most
//    1 + ceil((S - 1) / m) pairs, as every pair has m entries or more; with
//    Ctot <= raw + B H m and m >= raw / ((DF_MAX_PAIRS - 1) Ga - B H) that
//    is at most DF_MAX_PAIRS.  The host checks (DF_MAX_PAIRS - 1) Ga >= 2 B H,
//    so m <= max nk_b and Ctot <= B H max nk_b, and keeps Ctot Ga < 2^31.
// With equal lengths m <= nk_b, so nothing is padded.
struct AttnSched {
  int nk[8];
  int ne[8];
  int pre[9];
  int L[8];
  int Ga;
};
__host__ __device__ __forceinline__ int attn_ctas(int G, int H) {
  return G < (DF_CMAX - 1) * H ? G : (DF_CMAX - 1) * H;
}
__device__ __forceinline__ void attn_sched(const DfParams& p, int G, AttnSched& s) {
  int raw = 0;
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
    raw += p.H * s.nk[b];
  }
  s.Ga = attn_ctas(G, p.H);
  const int den = (DF_MAX_PAIRS - 1) * s.Ga - p.B * p.H;
  const int m = den > 0 ? max(1, (raw + den - 1) / den) : 1;
  s.pre[0] = 0;
  for (int b = 0; b < 8; ++b) {
    s.ne[b] = b < p.B ? max(s.nk[b], m) : 0;
    s.pre[b + 1] = s.pre[b] + p.H * s.ne[b];
  }
}
__device__ __forceinline__ void attn_entry(const AttnSched& s, int c, int& b, int& h, int& kc) {
  b = 0;
  while (b < 7 && c >= s.pre[b + 1]) ++b;
  const int r = c - s.pre[b];
  h = r / s.ne[b];
  kc = r - h * s.ne[b];
}
// This CTA's attention entries [c0, c1) (empty past the first Ga CTAs;
// 32-bit: the host keeps entries x Ga below 2^31).
__device__ __forceinline__ void attn_share(const AttnSched& s, int g, int& c0, int& c1) {
  if (g < s.Ga) {
    share(s.pre[8], s.Ga, g, c0, c1);
  } else {
    c0 = c1 = 0;
  }
}

// Contributors of a tile (or attention pair) are the CTAs whose shares hold
// its entries: a contiguous CTA range.  A unit of the contributor table is
// u[0] = count, u[1..] = partial slot indices (gg * DF_MAX_SU + su).

// Tile t of GEMV stage q.  False if the slots do not fit the table.
__host__ __device__ __forceinline__ bool tile_slots(const DfPhase& q, int t, int G, short* u) {
  const int Ctot = q.T * q.nk;
  const int gf = owner_of(t * q.nk, Ctot, G), gl = owner_of(t * q.nk + q.nk - 1, Ctot, G);
  int n = 0;
  bool ok = true;
  for (int gg = gf; gg <= gl; ++gg) {
    if (Ctot < G && !share_nonempty(Ctot, G, gg)) continue;
    const int su = t - (gg * Ctot / G) / q.nk;
    if (su < 0 || su >= DF_MAX_SU || n >= DF_CMAX) { ok = false; continue; }
    u[1 + n++] = (short)(gg * DF_MAX_SU + su);
  }
  u[0] = (short)n;
  return ok;
}

// Attention pair (b, h): every CTA whose share meets the pair's entries
// (empty ones included) writes one partial of it.
__device__ __forceinline__ bool pair_slots(const AttnSched& s, int H, int b, int h, short* u) {
  const int Ctot = s.pre[8], G = s.Ga;
  const int e0 = s.pre[b] + h * s.ne[b];
  const int gf = owner_of(e0, Ctot, G), gl = owner_of(e0 + s.ne[b] - 1, Ctot, G);
  int n = 0;
  bool ok = true;
  for (int gg = gf; gg <= gl; ++gg) {
    if (Ctot < G && !share_nonempty(Ctot, G, gg)) continue;
    int b2, h2, k2;
    attn_entry(s, gg * Ctot / G, b2, h2, k2);
    const int su = b * H + h - (b2 * H + h2);
    if (su < 0 || su >= DF_MAX_SU || n >= DF_CMAX) { ok = false; continue; }
    u[1 + n++] = (short)(gg * DF_MAX_SU + su);
  }
  u[0] = (short)n;
  return ok;
}

__device__ __forceinline__ void add4(float4& a, const float4& b, float w = 1.f) {
  a.x = fmaf(w, b.x, a.x); a.y = fmaf(w, b.y, a.y); a.z = fmaf(w, b.z, a.z); a.w = fmaf(w, b.w, a.w);
}
// Sums of 4 consecutive floats over two units' partial slots (s0 at idx0
// over u0; s1 at idx1 over u1 when has1), weighted by w0 / w1 when given.
// Slots are added in CTA order, so every reader gets the same bits; the
// loads of both sums are issued before any add, four slots at a time.
__device__ __forceinline__ void gather4x2(const float* buf, const short* u0, int idx0, const float* w0,
                                          const short* u1, int idx1, const float* w1, bool has1,
                                          float4& s0, float4& s1) {
  s0 = make_float4(0.f, 0.f, 0.f, 0.f);
  s1 = s0;
  const int n0 = u0[0], n1 = has1 ? u1[0] : 0;
  const int n = n0 > n1 ? n0 : n1;
  for (int c0 = 0; c0 < n; c0 += 4) {
    float4 a[4], b[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      a[c] = c0 + c < n0
                 ? __ldcg(reinterpret_cast<const float4*>(buf + (long long)u0[1 + c0 + c] * DF_PART_STRIDE + idx0))
                 : make_float4(0.f, 0.f, 0.f, 0.f);
      b[c] = c0 + c < n1
                 ? __ldcg(reinterpret_cast<const float4*>(buf + (long long)u1[1 + c0 + c] * DF_PART_STRIDE + idx1))
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (c0 + c < n0) add4(s0, a[c], w0 ? w0[c0 + c] : 1.f);
      if (c0 + c < n1) add4(s1, b[c], w1 ? w1[c0 + c] : 1.f);
    }
  }
}
// Softmax merge of one attention pair's (m, l, o) partials for dims
// [dim, dim + 4): an online merge in contributor (CTA) order, so every reader
// gets the same bits; loads four contributors at a time.
__device__ __forceinline__ float4 attn_gather4(const float* buf, const short* u, int dim) {
  const int n = u[0];
  float M = -INFINITY, Ls = 0.f;
  float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c0 = 0; c0 < n; c0 += 4) {
    float mc[4], lc[4];
    float4 oc[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      mc[c] = -INFINITY;
      lc[c] = 0.f;
      oc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c0 + c < n) {
        const float* ps = buf + (long long)u[1 + c0 + c] * DF_PART_STRIDE;
        mc[c] = __ldcg(ps);
        lc[c] = __ldcg(ps + 1);
        oc[c] = __ldcg(reinterpret_cast<const float4*>(ps + 4 + dim));
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (mc[c] == -INFINITY) continue;
      const float Mn = fmaxf(M, mc[c]);
      const float a = M == -INFINITY ? 0.f : ex2_approx(M - Mn), b = ex2_approx(mc[c] - Mn);
      Ls = Ls * a + lc[c] * b;
      O = make_float4(O.x * a + oc[c].x * b, O.y * a + oc[c].y * b, O.z * a + oc[c].z * b, O.w * a + oc[c].w * b);
      M = Mn;
    }
  }
  const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
  return make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
}

// Sum of 4 consecutive floats at idx over one unit's partial slots, in CTA
// order; up to eight slots' loads in flight together.
__device__ __forceinline__ float4 gather4_one(const float* buf, const short* u, int idx) {
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  const int n = u[0];
  for (int c0 = 0; c0 < n; c0 += 8) {
    float4 a[8];
#pragma unroll
    for (int c = 0; c < 8; ++c)
      a[c] = c0 + c < n ? __ldcg(reinterpret_cast<const float4*>(buf + (long long)u[1 + c0 + c] * DF_PART_STRIDE + idx))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      if (c0 + c < n) add4(s, a[c]);
  }
  return s;
}

template <int MT>
__device__ __forceinline__ void add_sq(float (&ssq)[MT], int m, const float4& v) {
#pragma unroll
  for (int mm = 0; mm < MT; ++mm)
    if (mm == m) ssq[mm] += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
}

// v * g[j .. j + 3] (bf16 gains)
__device__ __forceinline__ float4 gain4(float4 v, const bf16* g, int j) {
  const uint2 gr = __ldg(reinterpret_cast<const uint2*>(g + j));
  return make_float4(v.x * bf_lo(gr.x), v.y * bf_hi(gr.x), v.z * bf_lo(gr.y), v.w * bf_hi(gr.y));
}
__device__ __forceinline__ float4 round4(float4 v) {
  return make_float4(bf_round(v.x), bf_round(v.y), bf_round(v.z), bf_round(v.w));
}

// (a0, a1) += x * (y0, y1): one packed fp32x2 FMA (sm_100).
__device__ __forceinline__ void ffma2(float& a0, float& a1, float x, float y0, float y1) {
  asm("{\n\t.reg .b64 acc, xx, yy;\n\t"
      "mov.b64 acc, {%0, %1};\n\t"
      "mov.b64 xx, {%2, %2};\n\t"
      "mov.b64 yy, {%3, %4};\n\t"
      "fma.rn.f32x2 acc, xx, yy, acc;\n\t"
      "mov.b64 {%0, %1}, acc;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(x), "f"(y0), "f"(y1));
}

// acc[m][0..3] += A[m][kk] * W[kk][4 columns] over this lane's rows of a
// ring entry.  w points at the warp's region of the entry: 16-byte pieces
// (rows 2p and 2p + 1 of the warp's 4 columns), piece p = 32 i + lane, so
// every load of the warp reads 512 consecutive bytes.  a points at the
// entry's input chunk (row m at m * df_acols(MT)).  FULL: all 256 rows are
// valid; else pieces at or beyond kn / 2 are skipped (kn is even).
template <int MT, bool FULL>
__device__ __forceinline__ void entry_mac(float (&acc)[MT][4], const uint8_t* w, const float* a, int kn,
                                          int lane) {
  uint4 u[4];
  float2 av[4][MT];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int pc = 32 * i + lane;
    const bool valid = FULL || 2 * pc < kn;
    u[i] = valid ? *reinterpret_cast<const uint4*>(w + pc * 16) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int m = 0; m < MT; ++m)
      av[i][m] = valid ? *reinterpret_cast<const float2*>(a + m * df_acols(MT) + 2 * pc) : make_float2(0.f, 0.f);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float w0[4] = {bf_lo(u[i].x), bf_hi(u[i].x), bf_lo(u[i].y), bf_hi(u[i].y)};
    const float w1[4] = {bf_lo(u[i].z), bf_hi(u[i].z), bf_lo(u[i].w), bf_hi(u[i].w)};
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      ffma2(acc[m][0], acc[m][1], av[i][m].x, w0[0], w0[1]);
      ffma2(acc[m][2], acc[m][3], av[i][m].x, w0[2], w0[3]);
      ffma2(acc[m][0], acc[m][1], av[i][m].y, w1[0], w1[1]);
      ffma2(acc[m][2], acc[m][3], av[i][m].y, w1[2], w1[3]);
    }
  }
}

// Sum each of V values over the 32 lanes of a warp (V a power of 2, 4..16)
// as a reduce-scatter: rounds with lane masks 16, 8, ... halve the values a
// lane keeps, the rest are plain butterflies.  Returns the sum of value
// scatter_index(lane), identical on the lanes that share it.
template <int V>
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[V], int lane) {
#pragma unroll
  for (int n = V, s = 16; n > 1; n >>= 1, s >>= 1) {
    const bool hi = (lane & s) != 0;
#pragma unroll
    for (int j = 0; j < n / 2; ++j) {
      const float send = hi ? v[j] : v[j + n / 2];
      const float keep = hi ? v[j + n / 2] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  float r = v[0];
#pragma unroll
  for (int s = 16 / V; s >= 1; s >>= 1) r += __shfl_xor_sync(0xffffffffu, r, s);
  return r;
}
template <int V>
__device__ __forceinline__ int scatter_index(int lane) {
  int idx = 0;
#pragma unroll
  for (int n = V, s = 16; n > 1; n >>= 1, s >>= 1)
    if (lane & s) idx += n / 2;
  return idx;
}

// Asynchronous 16-byte global -> shared copy (completion: cp_async_wait).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <int MT>
__global__ void __launch_bounds__(DfCfg<MT>::THREADS, 1)
decode_layer_kernel(const __grid_constant__ DfParams p) {
  using C = DfCfg<MT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* slots = smem;
  float* abuf = reinterpret_cast<float*>(smem + C::NSLOT * C::SLOT);   // [MT][C::ACOLS]
  float* red = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(abuf) + C::ABUF_BYTES);
  float* scr = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(red) + C::RED_BYTES);
  uint8_t* misc = reinterpret_cast<uint8_t*>(scr) + C::SCR_BYTES;
  // Two schedule-record buffers: GEMV stage k reads buffer k & 1 while the
  // record of stage k + 1 lands in the other one (asynchronous copy).
  SchedRec* const srec_buf = reinterpret_cast<SchedRec*>(misc);
  SchedRec* srec = srec_buf;  // this CTA's record of the current stage
  int* clist = srec->clist;
  short* utab = &srec->utab[0][0];
  AttnSched* s_as = reinterpret_cast<AttnSched*>(misc + 2 * sizeof(SchedRec) + 64);  // attention schedule
  static_assert(C::RED_BYTES >= C::CW * MT * 4, "norm sums area");
  static_assert(2 * sizeof(SchedRec) + 64 + sizeof(AttnSched) <= C::MISC_BYTES, "misc shared area");
  uint64_t* full = reinterpret_cast<uint64_t*>(misc + C::MISC_BYTES);
  uint64_t* empty = full + C::NSLOT;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + C::NSLOT);
  // consumers' copy of the current layer's record tail: pack, sched,
  // k_cache, v_cache, then the stage table
  // (layer l reads copy l & 1; the next layer's lands in the other one)
  uint8_t* const s_lyb_buf = reinterpret_cast<uint8_t*>(full) + C::BAR_BYTES;
  uint8_t* s_lyb = s_lyb_buf;
  DfPhase* s_ph = reinterpret_cast<DfPhase*>(s_lyb + (offsetof(DfLayer, ph) - offsetof(DfLayer, pack)));
  constexpr int LYQ = (int)(offsetof(DfLayer, ph) + sizeof(DfPhase) * DF_NPHASE - offsetof(DfLayer, pack)) / 16;
  static_assert(LYQ * 16 <= C::PH_BYTES / 2 && offsetof(DfLayer, pack) % 16 == 0 &&
                    (offsetof(DfLayer, ph) + sizeof(DfPhase) * DF_NPHASE - offsetof(DfLayer, pack)) % 16 == 0,
                "layer record tail exceeds its shared copy");

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, g = blockIdx.x;
  const long long half = (long long)G * DF_MAX_SU * DF_PART_STRIDE;

  auto layer_of = [&](int l) -> const DfLayer* { return p.layers ? p.layers + l : &p.inl; };
  if (tid == 0) {
    for (int s = 0; s < C::NSLOT; ++s) {
      tc::mbar_init(full + s, 1);
      tc::mbar_init(empty + s, C::CW);
    }
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  if (warp == C::CW) {
    // =================================================== producer ==========
    // Fills every ring entry in order, layer after layer: pack entries of the
    // GEMV stages (the next layer's while the current one finishes), 64-key
    // cache chunks of the attention stages.
    if (lane == 0) {
      // L2 prefetch cursor (layer, stage, entry), PF pack entries ahead
      constexpr int PF = 2;
      const uint64_t pol_last = policy_evict_last();
      int pf_l = 0, pf_s = -1, pf_c = 0, pf_c1 = 0;
      auto pf_step = [&]() {
        while (pf_c >= pf_c1) {
          if (pf_l >= p.nlayer) return;
          if (++pf_s >= DF_NPHASE) {
            pf_s = 0;
            if (++pf_l >= p.nlayer) return;
          }
          const DfPhase& q = layer_of(pf_l)->ph[pf_s];
          if (q.type != DF_GEMV) { pf_c = pf_c1 = 0; continue; }
          share(q.T * q.nk, G, g, pf_c, pf_c1);
        }
        const DfLayer* Lq = layer_of(pf_l);
        const DfPhase& q = Lq->ph[pf_s];
        const int t = pf_c / q.nk, kc = pf_c - t * q.nk;
        const int kn = min(DF_KC, q.K - kc * DF_KC);
        const uint8_t* pe = Lq->pack + q.pack_off + (long long)t * q.K * 128 + (long long)kc * 32768;
        if (q.shared)
          prefetch_l2_bulk_hint(pe, (uint32_t)kn * 128u, pol_last);
        else
          prefetch_l2_bulk(pe, (uint32_t)kn * 128u);
        ++pf_c;
      };
      for (int i = 0; i < PF; ++i) pf_step();
      int seq = 0;
      bool waited = false, ok = true;
      AttnSched s;
      int a0 = 0, a1 = 0;
      const int NB = p.D >> 6;
      for (int l = 0; l < p.nlayer && ok && !*abort_flag; ++l) {
        const DfLayer* Ly = layer_of(l);
        for (int ph_i = 0; ph_i < DF_NPHASE && ok && !*abort_flag; ++ph_i) {
          const DfPhase& ph = Ly->ph[ph_i];
          if (ph_i == 1) {
            // History lengths are fixed for this step: the attention
            // schedule (and this CTA's share of it) once the previous
            // kernel is done.  The cache chunks are not prefetched into L2
            // here: that extra HBM traffic during the q/k/v stage slowed
            // the stage more than it sped up the attention stage.
            if (!waited) {
              pdl_wait();
              waited = true;
              attn_sched(p, G, s);
              attn_share(s, g, a0, a1);
            }
            tc::tma_prefetch_desc(&Ly->kmap);
            tc::tma_prefetch_desc(&Ly->vmap);
          }
          if (ph.type == DF_ATTN) {
            // K/V chunks of the dense cache (rows before the current position
            // are fixed for this step; the current row is taken from q/k/v)
            for (int c = a0; c < a1; ++c) {
              int b, h, kc;
              attn_entry(s, c, b, h, kc);
              if (kc >= s.nk[b]) continue;  // padding: no ring entry
              const int slot = seq % C::NSLOT;
              const uint32_t par = (uint32_t)(seq / C::NSLOT) & 1u;
              ++seq;
              if (!tc::mbar_wait_sleep(empty + slot, par ^ 1u, abort_flag, p.status)) { ok = false; break; }
              uint8_t* base = slots + slot * C::SLOT;
              tc::mbar_expect_tx(full + slot, (uint32_t)(2 * NB * 8192));
              const int row = b * p.S_max + kc * 64;
              for (int bx = 0; bx < NB; ++bx) {
                tc::tma_load_2d(base + bx * 8192, &Ly->kmap, full + slot, h * p.D + 64 * bx, row);
                tc::tma_load_2d(base + 16384 + bx * 8192, &Ly->vmap, full + slot, h * p.D + 64 * bx, row);
              }
            }
            continue;
          }
          int c0, c1;
          share(ph.T * ph.nk, G, g, c0, c1);
          for (int c = c0; c < c1; ++c, ++seq) {
            const int slot = seq % C::NSLOT;
            const uint32_t par = (uint32_t)(seq / C::NSLOT) & 1u;
            if (!tc::mbar_wait_sleep(empty + slot, par ^ 1u, abort_flag, p.status)) { ok = false; break; }
            const int t = c / ph.nk, kc = c - t * ph.nk;
            const uint32_t bytes = (uint32_t)min(DF_KC, ph.K - kc * DF_KC) * 128u;
            const uint8_t* e = Ly->pack + ph.pack_off + (long long)t * ph.K * 128 + (long long)kc * 32768;
            tc::mbar_expect_tx(full + slot, bytes);
            if (ph.shared)
              bulk_g2s_hint(slots + slot * C::SLOT, e, bytes, full + slot, pol_last);
            else
              bulk_g2s(slots + slot * C::SLOT, e, bytes, full + slot);
            pf_step();
          }
        }
      }
      if (*abort_flag) {
        const long long t0 = clock64();  // let copies in flight land
        while (clock64() - t0 < 2000000) {}
      }
    }
  } else {
    // ================================================= consumers ==========
    pdl_wait();
    if (tid == 0) attn_sched(p, G, *s_as);  // lengths are fixed for the launch
    // Consumer warp w owns columns 4 w .. 4 w + 3 of every ring entry (box
    // w / 8) over all of the entry's rows: a tile's column sums need no
    // exchange between warps.
    const int box = warp >> 3;
    int seq = 0;
    // Schedule record of the next GEMV stage, one 16-byte piece per thread
    // (stage 0 after the first layer uses the previous layer's record 10).
    // All of it comes from the current layer's records (sched_cur); the
    // next layer's record tail is loaded into registers during the last stage.
    bool rec_ready = false, ly_ready = false;
    int gidx = 0;  // GEMV stages done in this launch: the current one reads srec_buf[gidx & 1]
    const SchedRec* sched_cur = nullptr;
    auto rec_fetch = [&](int rl, int rph, int buf) {
      static_assert(sizeof(SchedRec) / 16 <= C::CT, "one 16-byte piece of the record per thread");
      const SchedRec* r = sched_cur + (long long)((rph == 0 && rl > 0) ? DF_NPHASE + 1 : rph) * G;
      SchedRec* dst = srec_buf + buf;
      if (tid < (int)(sizeof(SchedRec) / 16))
        cp_async16(reinterpret_cast<uint4*>(dst) + tid, reinterpret_cast<const uint4*>(r + g) + tid);
      cp_async_commit();
      rec_ready = true;
    };
    // layers after the first come from the device array p.layers
    auto ly_fetch = [&](int rl) {
      if (tid < LYQ)
        cp_async16(s_lyb_buf + (rl & 1) * (C::PH_BYTES / 2) + tid * 16,
                   reinterpret_cast<const uint4*>(&p.layers[rl].pack) + tid);
      cp_async_commit();
      ly_ready = true;
    };
    // record of the GEMV stage after (rl, rph) into buffer buf
    auto next_gemv_stage = [&](int rl, int rph, int buf) {
      ++rph;
      if (rph < DF_NPHASE && s_ph[rph].type != DF_GEMV) ++rph;
      if (rph >= DF_NPHASE) { rph = 0; ++rl; }
      if (rl < p.nlayer) {
        rec_fetch(rl, rph, buf);
        if (rph == 0) ly_fetch(rl);
      }
    };
    for (int l = 0; l < p.nlayer; ++l) {
    {
      // this layer's pointers and stage table, read in every inner loop
      consumer_sync<C::CT>();
      s_lyb = s_lyb_buf + (l & 1) * (C::PH_BYTES / 2);
      s_ph = reinterpret_cast<DfPhase*>(s_lyb + (offsetof(DfLayer, ph) - offsetof(DfLayer, pack)));
      if (l == 0) {
        if (tid < LYQ) reinterpret_cast<uint4*>(s_lyb)[tid] = reinterpret_cast<const uint4*>(&layer_of(0)->pack)[tid];
      } else {
        if (!ly_ready) ly_fetch(l);
        cp_async_wait();
      }
      ly_ready = false;
      consumer_sync<C::CT>();
      sched_cur = *reinterpret_cast<const SchedRec* const*>(s_lyb + (offsetof(DfLayer, sched) - offsetof(DfLayer, pack)));
    }
    for (int ph_i = 0; ph_i < DF_NPHASE; ++ph_i) {
      const DfPhase& ph = s_ph[ph_i];
      const int gs = l * DF_NPHASE + ph_i;  // global stage index
      float* part_cur = p.part + (gs & 1) * half;
      const float* part_prev = p.part + ((gs + 1) & 1) * half;
      // the previous stage is complete on every CTA once its counter
      // (accumulated over the layers) reaches prev_target
      const int prev_ctr = ph_i > 0 ? ph_i - 1 : DF_NPHASE - 1;
      const int prev_target = G * (ph_i > 0 ? l + 1 : l);
      DF_TRACE(l, ph_i, 0);
      if (ph.type == DF_GEMV) {
        const int src = (ph_i == 0 && l > 0) ? SRC_XOUT : ph.src;
        const int Ctot = ph.T * ph.nk;
        int c0, c1;
        share(Ctot, G, g, c0, c1);
        const int nseg = ph.map == MAP_SWIGLU ? 2 : 1;
        const bool xin = src == SRC_X || src == SRC_XMID || src == SRC_XOUT;
        // this CTA's schedule record of the stage (static: from the pack),
        // copied while the previous stage ran
        srec = srec_buf + (gidx & 1);
        clist = srec->clist;
        utab = &srec->utab[0][0];
        if (!rec_ready) rec_fetch(l, ph_i, gidx & 1);
        cp_async_wait();
        rec_ready = false;
        consumer_sync<C::CT>();

        // ---- the stage input, built from what the previous stage left ----
        // (1) contributor table: one unit per previous-stage tile (or
        // attention pair) that this CTA's input chunks draw on; static ones
        // come with the record, attention pairs depend on the lengths.
        const int n = srec->n;
        const int hpc = DF_KC / p.D;  // heads per 256-column chunk
        int nunits = srec->nunits;
        if (src == SRC_ATT) {
          nunits = n * MT * hpc;
          if (nunits > DF_MAX_UNITS) {
            if (tid == 0) atomicExch(p.status, DEV_STATUS_SCHEDULE);
            nunits = 0;
          }
          const AttnSched& s = *s_as;
          for (int ui = tid; ui < nunits; ui += C::CT) {
            short* u = utab + ui * 16;
            u[0] = 0;
            const int j = ui % hpc, r2 = ui / hpc, m = r2 % MT, ci = r2 / MT;
            const int hh = (clist[ci] & 255) * DF_KC / p.D + j;
            if (m < p.B && hh < p.H && !pair_slots(s, p.H, m, hh, u)) atomicExch(p.status, DEV_STATUS_SCHEDULE);
          }
        }
        float ssq[MT];  // RMSNorm: sum of squares of this thread's input values
#pragma unroll
        for (int m = 0; m < MT; ++m) ssq[m] = 0.f;
        if (xin) {
          // x (the layer input, complete before this stage) into the input
          // rows; zero rows past B.  SRC_XOUT: the previous layer's x'
          // (stored at its stage 5, several barriers ago), to which the
          // partials of z V_dn are added after the barrier.
          const int d4 = p.d >> 2;
          const bf16* xsrc = src == SRC_XOUT ? p.xm : p.x;
          for (int e = tid; e < MT * d4; e += C::CT) {
            const int m = e / d4, j = (e - m * d4) * 4;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (m < p.B) {
              const uint2 raw = __ldcg(reinterpret_cast<const uint2*>(xsrc + (long long)m * p.d + j));
              v = make_float4(bf_lo(raw.x), bf_hi(raw.x), bf_lo(raw.y), bf_hi(raw.y));
              if (src == SRC_X) {
                add_sq<MT>(ssq, m, v);
                if (ph.norm) v = gain4(v, ph.norm_g, j);
              }
            }
            *reinterpret_cast<float4*>(abuf + m * C::ACOLS + j) = v;
          }
        }
        if (ph.norm) {
          // the norm gains, into L1 for the scaling after the barrier
          for (int o = tid * 64; o < p.d; o += C::CT * 64)
            asm volatile("prefetch.global.L1 [%0];" ::"l"(ph.norm_g + o));
        }
        // ---- wait for the previous stage on every CTA ----
        if ((ph_i > 0 || l > 0) && tid == 0) grid_wait(p.bar + prev_ctr, prev_target, abort_flag, p.status);
        DF_TRACE(l, ph_i, 1);
        consumer_sync<C::CT>();
        // (2) the input itself, 4 consecutive values per group, two groups
        // per thread and step (their loads in flight together)
        if ((src == SRC_XMID || src == SRC_XOUT) && nunits) {
          // x' = x + (z V_o) (SRC_XMID), or the previous layer's output
          // x = x' + (z V_dn) (SRC_XOUT), rounded as the residual stream is
          // stored; the owners of its 64-column tiles also store it
          const int d4 = p.d >> 2, tot = p.B * d4;
          for (int e0 = tid; e0 < tot; e0 += 2 * C::CT) {
            const int e1 = e0 + C::CT;
            const bool h1 = e1 < tot;
            const int m0 = e0 / d4, j0 = (e0 - m0 * d4) * 4;
            const int m1 = h1 ? e1 / d4 : 0, j1 = h1 ? (e1 - m1 * d4) * 4 : 0;
            float4 sp[2];
            gather4x2(part_prev, utab + (j0 >> 6) * 16, m0 * 64 + (j0 & 63), nullptr, utab + (j1 >> 6) * 16,
                      m1 * 64 + (j1 & 63), nullptr, h1, sp[0], sp[1]);
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
              if (k2 == 1 && !h1) continue;
              const int m = k2 ? m1 : m0, j = k2 ? j1 : j0;
              float4* a4 = reinterpret_cast<float4*>(abuf + m * C::ACOLS + j);
              float4 v = *a4;  // x (SRC_XMID) or the previous layer's x' (SRC_XOUT)
              add4(v, sp[k2]);
              v = round4(v);
              add_sq<MT>(ssq, m, v);
              *a4 = ph.norm ? gain4(v, ph.norm_g, j) : v;
              if ((j >> 6) % G == g) {
                uint2 o;
                o.x = pack_bf2(v.x, v.y);
                o.y = pack_bf2(v.z, v.w);
                *reinterpret_cast<uint2*>((src == SRC_XMID ? p.xm : p.x) + (long long)m * p.d + j) = o;
              }
            }
          }
        } else if (src == SRC_SWIGLU) {
          // h = SiLU(gate) * up; a SwiGLU tile holds 32 gate then 32 up columns
          const int tot = n * MT * 64;
          for (int e = tid; e < tot; e += C::CT) {
            const int i = (e & 63) * 4, m = (e >> 6) % MT, ci = (e >> 6) / MT;
            const int k = (clist[ci] & 255) * DF_KC + i;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (m < p.B && k < ph.K && nunits) {
              const short* u = utab + (ci * 8 + (i >> 5)) * 16;
              float4 gv, uv;
              gather4x2(part_prev, u, m * 64 + (k & 31), nullptr, u, m * 64 + (k & 31) + 32, nullptr, true, gv,
                        uv);
              v = round4(make_float4(gv.x / (1.f + expf(-gv.x)) * uv.x, gv.y / (1.f + expf(-gv.y)) * uv.y,
                                     gv.z / (1.f + expf(-gv.z)) * uv.z, gv.w / (1.f + expf(-gv.w)) * uv.w));
            }
            *reinterpret_cast<float4*>(abuf + m * C::ACOLS + ci * 256 + i) = v;
          }
        } else if (src == SRC_ATT) {
          // attention output: dims k % D .. + 3 of head k / D of row m
          const int tot = n * MT * 64;
          for (int e = tid; e < tot; e += C::CT) {
            const int i = (e & 63) * 4, m = (e >> 6) % MT, ci = (e >> 6) / MT;
            const int k = (clist[ci] & 255) * DF_KC + i;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (m < p.B && k < ph.K && nunits)
              v = round4(attn_gather4(part_prev, utab + ((ci * MT + m) * hpc + i / p.D) * 16, k % p.D));
            *reinterpret_cast<float4*>(abuf + m * C::ACOLS + ci * 256 + i) = v;
          }
        } else if (src == SRC_PART) {
          // fp32 rank activations z (plain column tiles of 64)
          const int tot = n * nseg * MT * 64;
          if (tot <= C::CT) {
            // at most one group per thread: all its slots' loads at once
            const int e = tid;
            if (e < tot) {
              const int i = (e & 63) * 4;
              int rest = e >> 6;
              const int m = rest % MT;
              rest /= MT;
              const int seg = rest % nseg, ci = rest / nseg;
              const int kc = clist[ci] & 255;
              const int k = kc * DF_KC + i;
              float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
              if (m < p.B && k < ph.K && nunits) {
                const int col = seg * ph.a_col2 + k, col0 = seg * ph.a_col2 + kc * DF_KC;
                v = gather4_one(part_prev, utab + ((ci * nseg + seg) * ph.ustride + (col >> 6) - (col0 >> 6)) * 16,
                                m * 64 + (col & 63));
              }
              *reinterpret_cast<float4*>(abuf + m * C::ACOLS + ci * 256 * nseg + seg * 256 + i) = v;
            }
          } else
          for (int e0 = tid; e0 < tot; e0 += 2 * C::CT) {
            const short* uu[2];
            const float* ww[2];
            int idx[2], dst[2];
            bool ok[2];
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
              const int e = e0 + k2 * C::CT;
              const int i = (e & 63) * 4;
              int rest = e >> 6;
              const int m = rest % MT;
              rest /= MT;
              const int seg = rest % nseg, ci = rest / nseg;
              const int kc = clist[ci < n ? ci : 0] & 255;
              const int k = kc * DF_KC + i;
              ok[k2] = e < tot && m < p.B && k < ph.K && nunits;
              dst[k2] = e < tot ? m * C::ACOLS + ci * 256 * nseg + seg * 256 + i : -1;
              uu[k2] = utab;
              ww[k2] = nullptr;
              idx[k2] = 0;
              if (!ok[k2]) continue;
              const int col = seg * ph.a_col2 + k, col0 = seg * ph.a_col2 + kc * DF_KC;
              uu[k2] = utab + ((ci * nseg + seg) * ph.ustride + (col >> 6) - (col0 >> 6)) * 16;
              idx[k2] = m * 64 + (col & 63);
            }
            float4 sv[2];
            if (ok[0] || ok[1]) {
              const bool sw = !ok[0];  // keep the live group first
              gather4x2(part_prev, uu[sw ? 1 : 0], idx[sw ? 1 : 0], ww[sw ? 1 : 0], uu[1], idx[1], ww[1],
                        ok[0] && ok[1], sv[sw ? 1 : 0], sv[1]);
            }
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
              if (dst[k2] < 0) continue;
              *reinterpret_cast<float4*>(abuf + dst[k2]) = ok[k2] ? sv[k2] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }
        }
        // RMSNorm: the input holds x * g; rstd(x) scales the column sums at
        // each tile's end.  Per-warp sums of squares go out with this barrier.
        if (ph.norm) {
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const float ss = warp_sum(ssq[m]);
            if (lane == 0) red[warp * MT + m] = ss;
          }
        }
        consumer_sync<C::CT>();
        float rstd[MT];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          rstd[m] = 1.f;
          if (ph.norm) {
            float ss = 0.f;
#pragma unroll
            for (int w = 0; w < C::CW; ++w) ss += red[w * MT + m];
            rstd[m] = rsqrtf(ss / (float)p.d + p.eps);
          }
        }

        DF_TRACE(l, ph_i, 2);
        next_gemv_stage(l, ph_i, (gidx + 1) & 1);  // its record loads under this stage's entries
        // ---- entries ----
        float acc[MT][4];
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[m][j] = 0.f;
        int su = 0;
        for (int c = c0; c < c1; ++c, ++seq) {
          const int slot = seq % C::NSLOT;
          const uint32_t par = (uint32_t)(seq / C::NSLOT) & 1u;
          tc::mbar_wait(full + slot, par, abort_flag, p.status);  // on abort: run on, results discarded
          const int t = c / ph.nk, kc = c - t * ph.nk;
          const int k0 = kc * DF_KC;
          const int kn = min(DF_KC, ph.K - k0);
          const uint8_t* w = slots + slot * C::SLOT + warp * 8 * kn;
          const float* ain = ph.norm ? abuf + k0
                                     : abuf + srec->chunk_of[c - c0] * 256 * nseg + (nseg == 2 ? box * 256 : 0);
          if (kn == DF_KC) entry_mac<MT, true>(acc, w, ain, kn, lane);
          else entry_mac<MT, false>(acc, w, ain, kn, lane);
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(empty + slot);

          const bool tile_end = (c == c1 - 1) || (kc == ph.nk - 1);
          if (!tile_end) continue;
          // ---- tile t done: the warp's 4 x MT column sums, reduced over
          // its lanes, go straight to this CTA's partial slot ----
          constexpr int V = 4 * MT;
          float v[V];
#pragma unroll
          for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int j = 0; j < 4; ++j) { v[m * 4 + j] = acc[m][j]; acc[m][j] = 0.f; }
          const float sum = warp_reduce_scatter<V>(v, lane);
          if (su < DF_MAX_SU) {
            if ((lane & (32 / V - 1)) == 0) {
              const int idx = scatter_index<V>(lane);
              float r = rstd[0];
#pragma unroll
              for (int m = 1; m < MT; ++m)
                if ((idx >> 2) == m) r = rstd[m];
              __stcg(part_cur + ((long long)g * DF_MAX_SU + su) * DF_PART_STRIDE + (idx >> 2) * 64 + warp * 4 +
                         (idx & 3),
                     sum * r);
            }
          } else if (lane == 0) {
            atomicExch(p.status, DEV_STATUS_SCHEDULE);
          }
          ++su;
        }
      } else {
        // ---------------------------------------------- attention stage --
        // (contributor tables in the previous GEMV stage's record buffer;
        // the next one's record lands in the other)
        srec = srec_buf + ((gidx + 1) & 1);
        clist = srec->clist;
        utab = &srec->utab[0][0];
        next_gemv_stage(l, ph_i, gidx & 1);
        const AttnSched& s = *s_as;
        const int Ctot = s.pre[8];
        int c0, c1;
        attn_share(s, g, c0, c1);
        const int D = p.D, hd = D >> 1, tph = D >> 6;
        int pf = 0, np = 0;
        if (c0 < c1) {
          int b0, h0, k0, b1, h1, k1;
          attn_entry(s, c0, b0, h0, k0);
          attn_entry(s, c1 - 1, b1, h1, k1);
          pf = b0 * p.H + h0;
          np = b1 * p.H + h1 - pf + 1;
        }
        if (np > DF_MAX_PAIRS) {
          if (tid == 0) atomicExch(p.status, DEV_STATUS_SCHEDULE);
          np = DF_MAX_PAIRS;
        }
        // q, k, v of this CTA's (batch, head) pairs from the stage-1 partials:
        // RoPE on q and k at the row's position, bf16 rounding as the cache
        // stores them.  The owner of a pair's last key chunk appends k, v.
        float* qkv = abuf;  // [np][3][D]
        {
          const DfPhase& q1 = s_ph[ph_i - 1];
          const int nunits = np * 3 * tph;  // one per stage-1 tile: (pair, q/k/v, tile of the head)
          for (int ui = tid; ui < nunits; ui += C::CT) {
            const int j = ui % tph, r2 = ui / tph, prob = r2 % 3, pair = pf + r2 / 3;
            const int h = pair % p.H;
            if (!tile_slots(q1, q1.tile_start[prob] + h * tph + j, G, utab + ui * 16))
              atomicExch(p.status, DEV_STATUS_SCHEDULE);
          }
          if (tid == 0) grid_wait(p.bar + prev_ctr, prev_target, abort_flag, p.status);
          DF_TRACE(l, ph_i, 1);
          consumer_sync<C::CT>();
          for (int e = tid; e < np * 3 * (hd >> 2); e += C::CT) {
            const int i = (e % (hd >> 2)) * 4;
            const int r2 = e / (hd >> 2);
            const int prob = r2 % 3, pr = r2 / 3;
            const int pair = pf + pr, b = pair / p.H, h = pair - b * p.H;
            const int pos = s.L[b] - 1;
            const short* u = utab + (r2 * tph + (i >> 5)) * 16;
            float4 lo, hi;
            gather4x2(part_prev, u, b * 64 + (i & 31), nullptr, u, b * 64 + (i & 31) + 32, nullptr, true, lo, hi);
            if (prob < 2) {
              const float4 cs = *reinterpret_cast<const float4*>(p.rope_cos + (long long)pos * hd + i);
              const float4 sn = *reinterpret_cast<const float4*>(p.rope_sin + (long long)pos * hd + i);
              const float4 l2 = make_float4(lo.x * cs.x - hi.x * sn.x, lo.y * cs.y - hi.y * sn.y,
                                            lo.z * cs.z - hi.z * sn.z, lo.w * cs.w - hi.w * sn.w);
              hi = make_float4(hi.x * cs.x + lo.x * sn.x, hi.y * cs.y + lo.y * sn.y, hi.z * cs.z + lo.z * sn.z,
                               hi.w * cs.w + lo.w * sn.w);
              lo = l2;
            }
            lo = round4(lo);
            hi = round4(hi);
            *reinterpret_cast<float4*>(qkv + (pr * 3 + prob) * D + i) = lo;
            *reinterpret_cast<float4*>(qkv + (pr * 3 + prob) * D + i + hd) = hi;
            if (prob > 0 && owner_of(s.pre[b] + h * s.ne[b] + s.nk[b] - 1, Ctot, s.Ga) == g) {
              bf16* dst = *reinterpret_cast<bf16* const*>(
                              s_lyb + (prob == 1 ? offsetof(DfLayer, k_cache) : offsetof(DfLayer, v_cache)) -
                              offsetof(DfLayer, pack)) + ((long long)b * p.S_max + pos) * (p.H * D) +
                          h * D;
              uint2 o;
              o.x = pack_bf2(lo.x, lo.y); o.y = pack_bf2(lo.z, lo.w);
              *reinterpret_cast<uint2*>(dst + i) = o;
              o.x = pack_bf2(hi.x, hi.y); o.y = pack_bf2(hi.z, hi.w);
              *reinterpret_cast<uint2*>(dst + i + hd) = o;
            }
          }
        }
        consumer_sync<C::CT>();
        DF_TRACE(l, ph_i, 2);

        // Each consumer warp owns KPW = 64 / CW keys of every 64-key entry;
        // LPK = 32 / KPW lanes share a key, each holding cpl 16-byte chunks
        // (8 dims each) of q, k, v and o.  A warp keeps its online-softmax
        // state (m, and l, o per lane group) over all entries of a pair.
        // The key at the current position comes from qkv (its cache row may
        // not be written yet).
        constexpr int KPW = 64 / C::CW;
        constexpr int LPK = 32 / KPW;
        constexpr int CPL_MAX = 128 / (LPK * 8);
        const int cpl = D / (LPK * 8);
        const int grp = lane / LPK, sl = lane % LPK;
        const int key_l = warp * KPW + grp;
        float* wm = scr;       // [CW]
        float* wl = scr + 32;  // [CW]
        float* wo = scr + 64;  // [CW][128]
        float qv[CPL_MAX * 8], ov[CPL_MAX * 8];
#pragma unroll
        for (int e = 0; e < CPL_MAX * 8; ++e) { qv[e] = 0.f; ov[e] = 0.f; }
        float m_w = -INFINITY, l_g = 0.f;
        int su = 0;
        for (int c = c0; c < c1; ++c) {
          int b, h, kc;
          attn_entry(s, c, b, h, kc);
          int pr = b * p.H + h - pf;
          pr = pr < np ? pr : np - 1;  // only past the schedule limit (flagged above)
          const int pair_last = s.pre[b] + h * s.ne[b] + s.ne[b] - 1;
          const float* qn = qkv + pr * 3 * D;
          if (c == c0 || kc == 0) {
            m_w = -INFINITY;
            l_g = 0.f;
#pragma unroll
            for (int cc = 0; cc < CPL_MAX; ++cc)
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                ov[cc * 8 + e] = 0.f;
                qv[cc * 8 + e] = cc < cpl ? qn[(sl * cpl + cc) * 8 + e] * p.scale_log2 : 0.f;
              }
          }
          if (kc < s.nk[b]) {  // padding entries hold no keys
            const int slot = seq % C::NSLOT;
            const uint32_t par = (uint32_t)(seq / C::NSLOT) & 1u;
            ++seq;
            tc::mbar_wait(full + slot, par, abort_flag, p.status);  // on abort: run on, results discarded
            const int L = s.L[b], pos = L - 1;
            const int key = kc * 64 + key_l;
            const uint8_t* kb = slots + slot * C::SLOT;
            const uint8_t* vb = kb + 16384;
            // two partial dots (even / odd dims) keep the FMA chains short
            float dot = 0.f, dot1 = 0.f;
            if (key == pos) {
#pragma unroll
              for (int cc = 0; cc < CPL_MAX; ++cc)
                if (cc < cpl)
#pragma unroll
                  for (int e = 0; e < 8; ++e) dot = fmaf(qv[cc * 8 + e], qn[D + (sl * cpl + cc) * 8 + e], dot);
            } else {
#pragma unroll
              for (int cc = 0; cc < CPL_MAX; ++cc)
                if (cc < cpl) {
                  const int gc = sl * cpl + cc;
                  const uint4 u = *reinterpret_cast<const uint4*>(kb + (gc >> 3) * 8192 + key_l * 128 +
                                                                  (((gc & 7) ^ (key_l & 7)) << 4));
                  const float kv[8] = {bf_lo(u.x), bf_hi(u.x), bf_lo(u.y), bf_hi(u.y),
                                       bf_lo(u.z), bf_hi(u.z), bf_lo(u.w), bf_hi(u.w)};
#pragma unroll
                  for (int e = 0; e < 8; e += 2) {
                    dot = fmaf(qv[cc * 8 + e], kv[e], dot);
                    dot1 = fmaf(qv[cc * 8 + e + 1], kv[e + 1], dot1);
                  }
                }
            }
            dot += dot1;
#pragma unroll
            for (int o = LPK / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            const float sc = key < L ? dot : -INFINITY;
            float mb = sc;
#pragma unroll
            for (int o = LPK; o < 32; o <<= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
            const float mn = fmaxf(m_w, mb);
            if (mn != -INFINITY) {  // warp-uniform
              const float corr = m_w == -INFINITY ? 0.f : ex2_approx(m_w - mn);
              const float pj = sc == -INFINITY ? 0.f : ex2_approx(sc - mn);
              l_g = l_g * corr + pj;
#pragma unroll
              for (int e = 0; e < CPL_MAX * 8; ++e) ov[e] *= corr;
              if (sc != -INFINITY) {
                if (key == pos) {
#pragma unroll
                  for (int cc = 0; cc < CPL_MAX; ++cc)
                    if (cc < cpl)
#pragma unroll
                      for (int e = 0; e < 8; ++e)
                        ov[cc * 8 + e] = fmaf(pj, qn[2 * D + (sl * cpl + cc) * 8 + e], ov[cc * 8 + e]);
                } else {
#pragma unroll
                  for (int cc = 0; cc < CPL_MAX; ++cc)
                    if (cc < cpl) {
                      const int gc = sl * cpl + cc;
                      const uint4 u = *reinterpret_cast<const uint4*>(vb + (gc >> 3) * 8192 + key_l * 128 +
                                                                      (((gc & 7) ^ (key_l & 7)) << 4));
                      const float vv[8] = {bf_lo(u.x), bf_hi(u.x), bf_lo(u.y), bf_hi(u.y),
                                           bf_lo(u.z), bf_hi(u.z), bf_lo(u.w), bf_hi(u.w)};
#pragma unroll
                      for (int e = 0; e < 8; ++e) ov[cc * 8 + e] = fmaf(pj, vv[e], ov[cc * 8 + e]);
                    }
                }
              }
              m_w = mn;
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(empty + slot);
          }

          if (c != c1 - 1 && c != pair_last) continue;
          // ---- merge the lane groups, then the warps; write this CTA's
          // (m, l, o) partial of the pair ----
          float lw = l_g;
#pragma unroll
          for (int o = LPK; o < 32; o <<= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
#pragma unroll
          for (int cc = 0; cc < CPL_MAX; ++cc)
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float v = ov[cc * 8 + e];
#pragma unroll
              for (int o = LPK; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
              if (grp == 0 && cc < cpl) wo[warp * 128 + (sl * cpl + cc) * 8 + e] = v;
            }
          if (lane == 0) { wm[warp] = m_w; wl[warp] = lw; }
          consumer_sync<C::CT>();
          float Mc = -INFINITY;
#pragma unroll
          for (int w2 = 0; w2 < C::CW; ++w2) Mc = fmaxf(Mc, wm[w2]);
          float Lc = 0.f, oc = 0.f;
#pragma unroll
          for (int w2 = 0; w2 < C::CW; ++w2) {
            const float wgt = (wm[w2] == -INFINITY) ? 0.f : ex2_approx(wm[w2] - Mc);
            Lc += wgt * wl[w2];
            if (tid < D) oc += wgt * wo[w2 * 128 + tid];
          }
          float* ps = su < DF_MAX_SU ? part_cur + ((long long)g * DF_MAX_SU + su) * DF_PART_STRIDE : nullptr;
          if (ps) {
            if (tid < D) __stcg(ps + 4 + tid, oc);
            if (tid == 0) { __stcg(ps, Mc); __stcg(ps + 1, Lc); }
          } else if (tid == 0) {
            atomicExch(p.status, DEV_STATUS_SCHEDULE);
          }
          consumer_sync<C::CT>();
          ++su;
        }
      }
      // ---- this CTA is done with stage ph_i ----
      if (ph.type == DF_GEMV) ++gidx;
      consumer_sync<C::CT>();
      DF_TRACE(l, ph_i, 3);
      // (the CTA barrier above orders every consumer's writes before this
      // thread's release, which is cumulative over them)
      if (tid == 0 && !(p.drop_arrival && g == 0 && l == 0 && ph_i == 0)) red_release_add(p.bar + ph_i, 1);
    }
    }  // layers
    // ---- final pass: x = x' + z V_dn of the last layer, this CTA's tiles ----
    if (tid == 0) grid_wait(p.bar + DF_NPHASE - 1, G * p.nlayer, abort_flag, p.status);
    consumer_sync<C::CT>();
    {
      const float* part8 = p.part + ((p.nlayer * DF_NPHASE - 1) & 1) * half;
      // record DF_NPHASE of the last layer: tiles g, g + G, ... of its last stage
      const int4* src =
          reinterpret_cast<const int4*>(layer_of(p.nlayer - 1)->sched + (long long)DF_NPHASE * G + g);
      for (int w = tid; w < (int)(sizeof(SchedRec) / 16); w += C::CT) reinterpret_cast<int4*>(srec)[w] = __ldg(src + w);
      consumer_sync<C::CT>();
      const int nt = srec->nunits;
      for (int e = tid; e < min(nt, DF_MAX_UNITS) * p.B * 16; e += C::CT) {
        const int c4 = (e & 15) * 4, m = (e >> 4) % p.B, ui = (e >> 4) / p.B;
        const long long o = (long long)m * p.d + (g + ui * G) * 64 + c4;
        const uint2 raw = __ldcg(reinterpret_cast<const uint2*>(p.xm + o));
        float4 v = make_float4(bf_lo(raw.x), bf_hi(raw.x), bf_lo(raw.y), bf_hi(raw.y));
        float4 sp, unused;
        gather4x2(part8, utab + ui * 16, m * 64 + c4, nullptr, utab, 0, nullptr, false, sp, unused);
        add4(v, sp);
        uint2 w;
        w.x = pack_bf2(v.x, v.y);
        w.y = pack_bf2(v.z, v.w);
        *reinterpret_cast<uint2*>(p.x + o) = w;
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

}  // namespace


namespace {

// ------------------------------------------------------------ the pack --
// Entry (t, kc) of a stage -- rows [256 kc, 256 kc + kn) of column tile t,
// 128 kn bytes at byte offset  stage_off + t * K * 128 + kc * 32768 -- holds
// 16 warp regions of 8 kn bytes.  Region w covers the entry's columns
// 4 w .. 4 w + 3 (box w / 8: entry columns 0..31 are box 0, 32..63 box 1) as
// kn / 2 pieces of 16 bytes; piece p holds rows 2p and 2p + 1 of those 4
// columns, row-major.  A box's 32 source columns (and, for the SwiGLU map,
// source rows) follow the stage's output map; columns at or beyond the
// factor's width are zero.
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
    const int wr = (int)(rem / (8LL * kn));  // consumer warp region
    const int pc = (int)((rem - (long long)wr * 8 * kn) >> 4);
    const int box = wr >> 3;
    int pi = 0;
    for (int j = 1; j < 3; ++j)
      if (j < st.nprob && t >= st.tile_start[j]) pi = j;
    const int tl = t - st.tile_start[pi];
    long long srow = k0 + 2 * pc;
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
    col += 4 * (wr & 7);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (col < st.N[pi]) {
      const bf16* r0 = st.src[pi] + srow * st.ld[pi] + col;
      const uint2 a0 = __ldg(reinterpret_cast<const uint2*>(r0));
      const uint2 a1 = __ldg(reinterpret_cast<const uint2*>(r0 + st.ld[pi]));
      v = make_uint4(a0.x, a0.y, a1.x, a1.y);
    }
    *reinterpret_cast<uint4*>(p.dst + byte) = v;
  }
}


// ------------------------------------------------------------------ host --

// Stage table of one fused decode layer; Q, if given, receives each stage's
// factor sources for the pack kernel.  Returns the pack size in bytes.
long long build_stages(const DecodeLayerDesc& L, DfPhase* P, PackStage* Q) {
  const int d = L.d, r = L.r, rf = L.r_f, f = L.f;
  memset(P, 0, sizeof(DfPhase) * DF_NPHASE);
  long long off = 0;
  auto gemv = [&](int i, int map, int src, int K, const bf16* const* srcm, const long long* ld) {
    DfPhase& ph = P[i];
    ph.type = DF_GEMV; ph.map = map; ph.src = src; ph.K = K;
    ph.nk = ceil_div(K, DF_KC);
    int T = 0;
    for (int j = 0; j < ph.nprob; ++j) {
      ph.tile_start[j] = T;
      T += (map == MAP_SWIGLU) ? ceil_div(ph.N[j], 32) : ceil_div(ph.N[j], 64);
    }
    for (int j = ph.nprob; j < 4; ++j) ph.tile_start[j] = T;
    ph.T = T;
    ph.pack_off = off;
    ph.ustride = part_ustride(ph);
    if (Q) {
      PackStage& q = Q[i];
      q.off = off; q.K = K; q.T = T; q.map = map; q.nprob = ph.nprob;
      q.w_row2 = map == MAP_SWIGLU ? rf : 0;
      for (int j = 0; j < 4; ++j) q.tile_start[j] = ph.tile_start[j];
      for (int j = 0; j < ph.nprob; ++j) { q.N[j] = ph.N[j]; q.src[j] = srcm[j]; q.ld[j] = ld[j]; }
    }
    off += (long long)T * K * 128;
  };
  // 0: z_qkv = rmsnorm(x) . [U_q | U_k | U_v]
  P[0].nprob = 3; P[0].norm = 1; P[0].norm_g = L.g1;
  for (int i = 0; i < 3; ++i) P[0].N[i] = r;
  { const long long ld[3] = {r, r, r}; gemv(0, MAP_PLAIN, SRC_X, d, L.U, ld); }
  // 1: q, k, v = z . V  (RoPE applied by the readers)
  P[1].nprob = 3;
  for (int i = 0; i < 3; ++i) P[1].N[i] = d;
  { const long long ld[3] = {d, d, d}; gemv(1, MAP_ROPE, SRC_PART, r, L.V, ld); }
  // 2: attention
  P[2].type = DF_ATTN;
  P[2].pack_off = off;
  // 3: z = att . U_o
  P[3].nprob = 1; P[3].N[0] = r;
  { const long long ld[1] = {r}; gemv(3, MAP_PLAIN, SRC_ATT, d, &L.U_o, ld); }
  // 4: x' = x + z . V_o  (residual added by the readers)
  P[4].nprob = 1; P[4].N[0] = d;
  { const long long ld[1] = {d}; gemv(4, MAP_PLAIN, SRC_PART, r, &L.V_o, ld); }
  // 5: z = rmsnorm(x') . U_gu
  P[5].nprob = 1; P[5].N[0] = 2 * rf; P[5].norm = 1; P[5].norm_g = L.g2;
  { const long long ld[1] = {2 * rf}; gemv(5, MAP_PLAIN, SRC_XMID, d, &L.U_gu, ld); }
  // 6: gate and up halves: z_g V_g and z_u V_u, 32 + 32 columns per tile
  P[6].nprob = 1; P[6].N[0] = f; P[6].a_col2 = rf;
  { const long long ld[1] = {f}; gemv(6, MAP_SWIGLU, SRC_PART, rf, &L.V_gu, ld); }
  // 7: z = h . U_dn, h = SiLU(gate) * up
  P[7].nprob = 1; P[7].N[0] = rf;
  { const long long ld[1] = {rf}; gemv(7, MAP_PLAIN, SRC_SWIGLU, f, &L.U_dn, ld); }
  // 8: x'' = x' + z . V_dn  (added in the final pass)
  P[8].nprob = 1; P[8].N[0] = d;
  { const long long ld[1] = {d}; gemv(8, MAP_PLAIN, SRC_PART, rf, &L.V_dn, ld); }
  return off;
}

// Schedule records of every (stage, CTA) -- see SchedRec.  Returns false if
// a CTA's share exceeds a record's fixed capacity.
bool build_sched(const DfPhase* P, int G, int d, SchedRec* R) {
  memset(R, 0, sizeof(SchedRec) * DF_NREC * G);
  for (int i = 0; i < DF_NPHASE; ++i) {
    const DfPhase& ph = P[i];
    if (ph.type != DF_GEMV) continue;
    const int Ctot = ph.T * ph.nk;
    const int nseg = ph.map == MAP_SWIGLU ? 2 : 1;
    const bool xin = ph.src == SRC_X || ph.src == SRC_XMID;
    for (int g = 0; g < G; ++g) {
      SchedRec& r = R[i * G + g];
      const int c0 = g * Ctot / G, c1 = (g + 1) * Ctot / G;
      if (c1 - c0 > DF_MAX_E) return false;
      if (!xin) {
        for (int c = c0; c < c1; ++c) {
          const int t = c / ph.nk, kc = c - t * ph.nk;
          int pi = 0;
          for (int j = 1; j < ph.nprob; ++j)
            if (t >= ph.tile_start[j]) pi = j;
          const int key = pi << 8 | kc;
          int ci = 0;
          while (ci < r.n && r.clist[ci] != key) ++ci;
          if (ci == r.n) {
            if (r.n == 16 || (r.n + 1) * 256 * nseg > DF_ABUF_WIDE) return false;
            r.clist[r.n++] = key;
          }
          r.chunk_of[c - c0] = (uint8_t)ci;
        }
      }
      const DfPhase& q = P[i > 0 ? i - 1 : 0];
      if (ph.src == SRC_XMID) {
        r.nunits = d >> 6;
        for (int t = 0; t < r.nunits; ++t)
          if (!tile_slots(P[4], t, G, r.utab[t])) return false;
      } else if (ph.src == SRC_PART) {
        const int us = ph.ustride;
        r.nunits = r.n * nseg * us;
        for (int ui = 0; ui < r.nunits; ++ui) {
          const int j = ui % us, cs = ui / us, seg = cs % nseg, ci = cs / nseg;
          const int pi = r.clist[ci] >> 8, kc = r.clist[ci] & 255;
          const int col0 = seg * ph.a_col2 + kc * DF_KC;
          const int kn = std::min(DF_KC, ph.K - kc * DF_KC);
          if ((col0 >> 6) + j <= (col0 + kn - 1) >> 6 &&
              !tile_slots(q, q.tile_start[pi] + (col0 >> 6) + j, G, r.utab[ui]))
            return false;
        }
      } else if (ph.src == SRC_SWIGLU) {
        r.nunits = r.n * 8;
        for (int ui = 0; ui < r.nunits; ++ui) {
          const int t = ((r.clist[ui >> 3] & 255) * DF_KC >> 5) + (ui & 7);
          if (t < q.T && !tile_slots(q, t, G, r.utab[ui])) return false;
        }
      }
      if (r.nunits > DF_MAX_UNITS) return false;
    }
  }
  // record 10: every tile of the last stage (the next layer's input)
  for (int g = 0; g < G; ++g) {
    SchedRec& r = R[(DF_NPHASE + 1) * G + g];
    r.nunits = d >> 6;
    if (r.nunits > DF_MAX_UNITS) return false;
    for (int t = 0; t < r.nunits; ++t)
      if (!tile_slots(P[DF_NPHASE - 1], t, G, r.utab[t])) return false;
  }
  // record 9, the final pass: tiles g, g + G, ... of the last stage
  for (int g = 0; g < G; ++g) {
    SchedRec& r = R[DF_NPHASE * G + g];
    for (int t = g; t < (d >> 6); t += G) {
      if (r.nunits == DF_MAX_UNITS || !tile_slots(P[DF_NPHASE - 1], t, G, r.utab[r.nunits])) return false;
      ++r.nunits;
    }
  }
  return true;
}

// Byte offset of the schedule records in a pack of `factor_bytes`.
long long sched_offset(long long factor_bytes) { return (factor_bytes + 127) / 128 * 128; }

// Whether every CTA's share of every GEMV stage stays within the kernel's
// fixed per-CTA limits (tiles touched, input chunks, contributor table).
bool stages_fit(const DfPhase* P, int G, int MT, int D) {
  for (int i = 0; i < DF_NPHASE; ++i) {
    const DfPhase& ph = P[i];
    if (ph.type != DF_GEMV) continue;
    if (ph.nk > DF_MAX_NK) return false;
    const int Ctot = ph.T * ph.nk;
    if ((long long)Ctot * G >= (1LL << 31)) return false;
    const int nseg = ph.map == MAP_SWIGLU ? 2 : 1;
    for (int g = 0; g < G; ++g) {
      const int c0 = g * Ctot / G, c1 = (g + 1) * Ctot / G;
      if (c0 >= c1) continue;
      if ((c1 - 1) / ph.nk - c0 / ph.nk + 1 > DF_MAX_SU) return false;
      if (ph.src == SRC_X || ph.src == SRC_XMID) continue;
      bool seen[3][DF_MAX_NK] = {};
      int n = 0;
      for (int c = c0; c < c1; ++c) {
        const int t = c / ph.nk, kc = c - t * ph.nk;
        int pi = 0;
        for (int j = 1; j < ph.nprob; ++j)
          if (t >= ph.tile_start[j]) pi = j;
        if (!seen[pi][kc]) { seen[pi][kc] = true; ++n; }
      }
      if (n * 256 * nseg > df_acols(MT)) return false;
      int units = 0;
      if (ph.src == SRC_PART) units = n * nseg * ph.ustride;
      else if (ph.src == SRC_SWIGLU) units = n * 8;
      else if (ph.src == SRC_ATT) units = n * MT * (DF_KC / D);
      if (units > DF_MAX_UNITS) return false;
    }
  }
  return true;
}

}  // namespace

int decode_fused_supported(int B, int d, int D, int r, int r_f) {
  return B >= 1 && B <= 4 && (D == 64 || D == 128) && d % 64 == 0 && d <= DF_ABUF_COLS && r % 8 == 0 &&
         r_f % 8 == 0;
}

long long decode_pack_bytes(const DecodeLayerDesc& L, int sm_count) {
  DfPhase P[DF_NPHASE];
  return sched_offset(build_stages(L, P, nullptr)) + (long long)sizeof(SchedRec) * DF_NREC * sm_count;
}

int decode_pack_launch(const DecodeLayerDesc& L, void* dst, long long bytes, int sm_count,
                       cudaStream_t stream) {
  DfPhase P[DF_NPHASE];
  PackParams pp;
  memset(&pp, 0, sizeof(pp));
  const long long need = build_stages(L, P, pp.st);
  const int G = sm_count;
  const long long soff = sched_offset(need);
  if (bytes < soff + (long long)sizeof(SchedRec) * DF_NREC * G) return FLASHSVD_ERR_INVALID_ARG;
  std::vector<SchedRec> rec((size_t)DF_NREC * G);
  if (!build_sched(P, G, L.d, rec.data())) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  // (pageable source: the copy is staged before this call returns)
  FSVD_CUDA(cudaMemcpyAsync(static_cast<uint8_t*>(dst) + soff, rec.data(), sizeof(SchedRec) * rec.size(),
                            cudaMemcpyHostToDevice, stream));
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

namespace {

// The kernel's view of one layer (caches, pack, schedule, stage table).
int fill_layer(const DecodeLayerDesc& L, bf16* kc, bf16* vc, int B, int S_max, int G, DfLayer* out,
               long long* algo_bytes) {
  if (!L.pack || !kc || !vc) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  if (!decode_fused_supported(B, L.d, L.D, L.r, L.r_f) || L.f % 8) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  // Attention: the schedule keeps each CTA within DF_MAX_PAIRS pairs for
  // any lengths when these hold (see AttnSched).
  const int Ga = attn_ctas(G, L.H);
  if ((DF_MAX_PAIRS - 1) * Ga < 2 * B * L.H) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  if ((long long)B * L.H * ((S_max + 63) / 64) * Ga >= (1LL << 31)) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  memset(out, 0, sizeof(DfLayer));
  const long long pack_bytes = build_stages(L, out->ph, nullptr);
  if (!stages_fit(out->ph, G, B <= 1 ? 1 : (B <= 2 ? 2 : 4), L.D)) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  out->pack = static_cast<const uint8_t*>(L.pack);
  // the pack holds the schedule records for this device's SM count
  out->sched = reinterpret_cast<const SchedRec*>(out->pack + sched_offset(pack_bytes));
  const long long HD = (long long)L.H * L.D;
  FSVD_TRY(encode_map(&out->kmap, kc, (long long)B * S_max, HD, HD, 64, 64, true));
  FSVD_TRY(encode_map(&out->vmap, vc, (long long)B * S_max, HD, HD, 64, 64, true));
  out->k_cache = kc;
  out->v_cache = vc;
  // factor bytes of the layer, and the cache bytes at the longest context
  const long long d = L.d, r = L.r, rf = L.r_f, f = L.f;
  *algo_bytes = 2 * (4 * 2 * d * r + d * 2 * rf + 2 * rf * f + f * rf + rf * d) + 2LL * 2 * B * S_max * HD;
  return FLASHSVD_OK;
}

void fill_common(DfParams& p, const DecodeLayerDesc& L, int B, int S_max, const int* seqlens, bf16* x,
                 bf16* xm, float* part, int* bar, int* done, int* status) {
  p.B = B; p.H = L.H; p.D = L.D; p.S_max = S_max; p.d = L.d;
  p.eps = L.eps;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)L.D);
  p.seqlens = seqlens;
  p.x = x; p.xm = xm;
  p.rope_cos = L.rope_cos; p.rope_sin = L.rope_sin;
  p.part = part; p.bar = bar; p.done = done; p.status = status;
  p.drop_arrival = g_df_drop_arrival.exchange(0);
}

}  // namespace

std::atomic<int> g_df_drop_arrival{0};

namespace {

int launch_df(const DfParams& p, int G, double bytes, cudaStream_t stream) {
  const LaunchTag tag{p.nlayer > 1 ? "decode_layers_fused" : "decode_layer_fused", bytes, 0.0};
#define FSVD_DF_LAUNCH(MT_)                                                                          \
  {                                                                                                  \
    auto kern = decode_layer_kernel<MT_>;                                                            \
    static SmemAttrOnce smem_once;                                                                   \
    FSVD_TRY(set_smem_once(smem_once, kern, DfCfg<MT_>::SMEM));                                      \
    return launch_pdl_coop(tag, kern, dim3(G), dim3(DfCfg<MT_>::THREADS), (size_t)DfCfg<MT_>::SMEM, stream, p); \
  }
  if (p.B <= 1) FSVD_DF_LAUNCH(1)
  if (p.B <= 2) FSVD_DF_LAUNCH(2)
  FSVD_DF_LAUNCH(4)
#undef FSVD_DF_LAUNCH
}

}  // namespace

int decode_fused_launch(const DecodeLayerDesc& L, bf16* x, bf16* kc, bf16* vc, const int* seqlens,
                        int B, int S_max, bf16* xm, float* part, long long part_floats, int* bar,
                        int* done, int* status, int sm_count, cudaStream_t stream) {
  const int G = sm_count;
  if (2LL * G * DF_MAX_SU * DF_PART_STRIDE > part_floats) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  DfParams p;
  memset(&p, 0, sizeof(p));
  long long bytes = 0;
  FSVD_TRY(fill_layer(L, kc, vc, B, S_max, G, &p.inl, &bytes));
  p.layers = nullptr;
  p.nlayer = 1;
  fill_common(p, L, B, S_max, seqlens, x, xm, part, bar, done, status);
  return launch_df(p, G, (double)bytes, stream);
}

struct DecodePlan {
  DfParams p;           // layers points at dev; per-launch fields set at launch
  DfLayer* dev = nullptr;
  DecodeLayerDesc first;
  int G = 0;
  double bytes = 0.0;
};

int decode_plan_create(const DecodeLayerDesc* layers, int n, bf16* const* k_caches, bf16* const* v_caches,
                       int B, int S_max, int sm_count, DecodePlan** out) {
  if (!layers || n <= 0 || !k_caches || !v_caches || !out) return FLASHSVD_ERR_INVALID_ARG;
  const int G = sm_count;
  std::vector<DfLayer> host((size_t)n);
  double bytes = 0.0;
  for (int i = 0; i < n; ++i) {
    const DecodeLayerDesc& L = layers[i];
    // model-level shapes and tables must agree across the layers
    if (L.d != layers[0].d || L.H != layers[0].H || L.D != layers[0].D || L.f != layers[0].f ||
        L.eps != layers[0].eps || L.rope_cos != layers[0].rope_cos || L.rope_sin != layers[0].rope_sin)
      return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
    long long b = 0;
    FSVD_TRY(fill_layer(L, k_caches[i], v_caches[i], B, S_max, G, &host[i], &b));
    bytes += (double)b;
  }
  // Shared bases ([v1.5] Methodology 1, Basis Sharing): a U stage whose
  // factor pointers equal those of an earlier layer (same stage shape)
  // reads that layer's pack entries, so every layer of the plan streams the
  // same bytes, which an L2 evict-last hint keeps on chip after the first;
  // their bytes count once per step.
  for (int i = 1; i < n; ++i) {
    const int ustage[4] = {0, 3, 5, 7};
    for (int u = 0; u < 4; ++u) {
      const int st = ustage[u];
      for (int j = 0; j < i; ++j) {
        const DecodeLayerDesc &A = layers[i], &Bj = layers[j];
        bool same = false;
        if (st == 0) same = A.U[0] == Bj.U[0] && A.U[1] == Bj.U[1] && A.U[2] == Bj.U[2] && A.r == Bj.r;
        if (st == 3) same = A.U_o == Bj.U_o && A.r == Bj.r;
        if (st == 5) same = A.U_gu == Bj.U_gu && A.r_f == Bj.r_f;
        if (st == 7) same = A.U_dn == Bj.U_dn && A.r_f == Bj.r_f;
        const DfPhase &pi = host[i].ph[st], &pj = host[j].ph[st];
        if (!same || pi.K != pj.K || pi.nk != pj.nk || pi.T != pj.T || pi.nprob != pj.nprob) continue;
        // pj.pack_off is relative to layer j's pack (itself maybe shared)
        host[i].ph[st].pack_off = (long long)((host[j].pack + pj.pack_off) - host[i].pack);
        host[i].ph[st].shared = 1;
        host[j].ph[st].shared = 1;
        bytes -= 2.0 * (double)pi.K * (pi.T * 64);
        break;
      }
    }
  }
  DecodePlan* plan = new DecodePlan();
  if (cudaMalloc(&plan->dev, sizeof(DfLayer) * n) != cudaSuccess) {
    delete plan;
    return FLASHSVD_ERR_NO_MEMORY;
  }
  const cudaError_t e = cudaMemcpy(plan->dev, host.data(), sizeof(DfLayer) * n, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(plan->dev);
    delete plan;
    return cuda_status(e);
  }
  memset(&plan->p, 0, sizeof(plan->p));
  plan->p.layers = plan->dev;
  plan->p.nlayer = n;
  plan->first = layers[0];
  plan->G = G;
  plan->bytes = bytes;
  plan->p.B = B;
  plan->p.S_max = S_max;
  *out = plan;
  return FLASHSVD_OK;
}

int decode_plan_launch(const DecodePlan* plan, bf16* x, const int* seqlens, bf16* xm, float* part,
                       long long part_floats, int* bar, int* done, int* status, cudaStream_t stream) {
  if (2LL * plan->G * DF_MAX_SU * DF_PART_STRIDE > part_floats) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  DfParams p = plan->p;
  fill_common(p, plan->first, plan->p.B, plan->p.S_max, seqlens, x, xm, part, bar, done, status);
  return launch_df(p, plan->G, plan->bytes, stream);
}

void decode_plan_destroy(DecodePlan* plan) {
  if (!plan) return;
  cudaFree(plan->dev);
  delete plan;
}

}  // namespace fsvd

#ifdef FLASHSVD_TRACE
// Trace builds only (not part of the public ABI): the stage timeline of the
// fused decode kernel's last launches, laid out as
// u64 [64 layers][9 stages][148 CTAs][2: ns, cycles][4 points].
extern "C" __attribute__((visibility("default"))) int flashsvd_trace_read(void* host, size_t bytes) {
  if (!host) return FLASHSVD_ERR_INVALID_ARG;
  const size_t n = bytes < sizeof(fsvd::g_df_trace) ? bytes : sizeof(fsvd::g_df_trace);
  return cudaMemcpyFromSymbol(host, fsvd::g_df_trace, n) == cudaSuccess ? FLASHSVD_OK : FLASHSVD_ERR_CUDA;
}
extern "C" __attribute__((visibility("default"))) int flashsvd_trace_clear(void) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, fsvd::g_df_trace) != cudaSuccess) return FLASHSVD_ERR_CUDA;
  return cudaMemset(p, 0, sizeof(fsvd::g_df_trace)) == cudaSuccess ? FLASHSVD_OK : FLASHSVD_ERR_CUDA;
}
#endif
