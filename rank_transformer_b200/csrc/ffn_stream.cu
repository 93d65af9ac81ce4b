// Streamed low-rank encoder FFN on tcgen05 ("FlashSVD: Memory-Efficient
// Inference with Streaming for Low-Rank Models", abstract: the FFN's
// intermediate activations are streamed through tiles instead of being
// materialised):
//     y = GELU(z1 . V1 + b1) . U2 . V2 + b2 + resid,   z1 = x . U1 (given)
// One persistent CTA per 128-row tile of M; the [M x f] activation never
// leaves the SM.  Per tile:
//   for each 128-column chunk c of f:
//     S[c & 1]  = z1 . V1[:, c]            (TMEM cols 0..127 / 128..255)
//     H[c & 1]  = bf16(GELU(S + b1[c]))    (epilogue warps -> swizzled smem)
//     acc2     += H . U2[c, :]             (TMEM cols 256 .. 256 + r2)
//   z2 = bf16(acc2) -> smem (over z1's area)
//   y[:, 256 p ..] = z2 . V2[:, 256 p ..] + b2 + resid   (TMEM cols 0..255)
// The MMA of chunk c + 1 overlaps the epilogue of chunk c (two S and two H
// buffers).  Warps: 0 TMA producer, 1 MMA issuer, 2..17 epilogue (four per
// TMEM lane quadrant, a quarter of the chunk's columns each).  All B operands stream through one ring of 32 KB
// slots in the order the MMA warp consumes them.  z1 is read once per tile
// from the rank scratch and its L2 lines are discarded after use, so z1 is
// never written back to HBM either.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace fsvd {
namespace {

constexpr int FS_NPART = 4;                // epilogue warps per TMEM lane quadrant
constexpr int FS_EPI = 4 * FS_NPART;       // epilogue warps
constexpr int FS_THREADS = 32 * (2 + FS_EPI);
constexpr int FS_CPW = 128 / FS_NPART;     // chunk columns per epilogue warp
constexpr int FS_STAGES = 3;
constexpr int FS_SLOT = 32768;           // one 64-row k-block of B, up to 256 columns
constexpr int FS_RMAX = 256;             // r1, r2 <= 256 (multiples of 64)
constexpr int FS_BLK = 128 * 64 * 2;     // one [128 x 64] bf16 A block, 16 KB
constexpr int FS_Z_OFF = 0;                                   // z1, later z2: FS_RMAX / 64 blocks
constexpr int FS_H_OFF = FS_Z_OFF + (FS_RMAX / 64) * FS_BLK;  // H[2]: 2 blocks each
constexpr int FS_RING_OFF = FS_H_OFF + 2 * 2 * FS_BLK;
constexpr int FS_BAR_OFF = FS_RING_OFF + FS_STAGES * FS_SLOT;
constexpr int FS_SMEM = 1024 + FS_BAR_OFF + 256;
static_assert(FS_SMEM <= 232448, "shared memory budget");
constexpr uint32_t FS_TMEM_COLS = 512;   // S[2] 0..255 (Y reuses them), acc2 256..511

struct FsArgs {
  int M, f, r1, r2, d;
  const bf16* z1; long long ldz;  // rank activations (their L2 lines are discarded after use)
  int discard;
  const bf16* b1;      // [f] or null
  const bf16* b2;      // [d] or null
  const bf16* resid;   // [M x d] or null (may alias y)
  bf16* y;             // [M x d]
  int* status;
};

__device__ __forceinline__ uint32_t pack2(float a, float b) { return pack_bf2(a, b); }

// (the library's erf-form GELU on value pairs, as in the GEMM epilogue)
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


__global__ void __launch_bounds__(FS_THREADS, 1)
ffn_stream_kernel(const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmV1,
                  const __grid_constant__ CUtensorMap tmU2, const __grid_constant__ CUtensorMap tmV2,
                  const __grid_constant__ FsArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + FS_BAR_OFF);  // [FS_STAGES]
  uint64_t* empty = full + FS_STAGES;                                // [FS_STAGES]
  uint64_t* z_full = empty + FS_STAGES;
  uint64_t* z_empty = z_full + 1;
  uint64_t* s_full = z_empty + 1;   // [2]
  uint64_t* s_empty = s_full + 2;   // [2]
  uint64_t* h_full = s_empty + 2;   // [2]
  uint64_t* h_empty = h_full + 2;   // [2]
  uint64_t* acc_full = h_empty + 2;
  uint64_t* z2_full = acc_full + 1;
  uint64_t* y_full = z2_full + 1;
  uint64_t* y_empty = y_full + 1;
  uint64_t* drain = y_empty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  static_assert(FS_STAGES * 2 + 16 <= 30, "barrier area");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = (a.M + 127) / 128;
  const int NC = (a.f + 127) / 128;     // f-chunks
  const int KB1 = a.r1 / 64, KB2 = a.r2 / 64;
  const int NP = (a.d + 255) / 256;     // output passes

  if (threadIdx.x == 0) {
    for (int s = 0; s < FS_STAGES; ++s) {
      tc::mbar_init(full + s, 1);
      tc::mbar_init(empty + s, 1);
    }
    tc::mbar_init(z_full, 1);
    tc::mbar_init(z_empty, 1);
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(s_full + b, 1);
      tc::mbar_init(s_empty + b, FS_EPI);
      tc::mbar_init(h_full + b, FS_EPI);
      tc::mbar_init(h_empty + b, 1);
    }
    tc::mbar_init(acc_full, 1);
    tc::mbar_init(z2_full, FS_EPI);
    tc::mbar_init(y_full, 1);
    tc::mbar_init(y_empty, FS_EPI);
    tc::mbar_init(drain, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tmZ);
    tc::tma_prefetch_desc(&tmV1);
    tc::tma_prefetch_desc(&tmU2);
    tc::tma_prefetch_desc(&tmV2);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_holder, FS_TMEM_COLS);
    tc::tmem_relinquish();
    tc::fence_before_sync();
  }
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;
  pdl_launch_dependents();
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      // one ring slot: nbox boxes of [64 rows x 64 cols] at (col0 + 64 j, row0)
      auto slot_load = [&](const CUtensorMap* tm, int nbox, int col0, int row0) -> bool {
        if (!tc::mbar_wait(empty + stage, phase ^ 1u, abort_flag, a.status)) return false;
        tc::mbar_expect_tx(full + stage, (uint32_t)(nbox * 8192));
        uint8_t* dst = smem + FS_RING_OFF + stage * FS_SLOT;
        for (int j = 0; j < nbox; ++j) tc::tma_load_2d(dst + j * 8192, tm, full + stage, col0 + 64 * j, row0);
        ++issued;
        if (++stage == FS_STAGES) { stage = 0; phase ^= 1u; }
        return true;
      };
      int it = 0;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++it) {
        const int m0 = t * 128;
        // z1 of this tile (its area holds the previous tile's z2 until that
        // tile's last MMA has completed)
        if (!tc::mbar_wait(z_empty, ((uint32_t)it & 1u) ^ 1u, abort_flag, a.status)) { ok = false; break; }
        tc::mbar_expect_tx(z_full, (uint32_t)(KB1 * FS_BLK));
        for (int kb = 0; kb < KB1; ++kb)
          tc::tma_load_2d(smem + FS_Z_OFF + kb * FS_BLK, &tmZ, z_full, kb * 64, m0);
        for (int c = 0; c <= NC && ok; ++c) {
          if (c < NC)  // V1[:, chunk c]: KB1 k-blocks of [64 x 128]
            for (int kb = 0; kb < KB1 && ok; ++kb) ok = slot_load(&tmV1, 2, c * 128, kb * 64);
          if (c >= 1)  // U2[chunk c-1, :]: 2 k-blocks of [64 x r2]
            for (int kb = 0; kb < 2 && ok; ++kb) ok = slot_load(&tmU2, KB2, 0, (c - 1) * 128 + kb * 64);
        }
        for (int p = 0; p < NP && ok; ++p)  // V2[:, 256 p ..]: KB2 k-blocks of [64 x 256]
          for (int kb = 0; kb < KB2 && ok; ++kb) ok = slot_load(&tmV2, 4, p * 256, kb * 64);
      }
      if (!ok) {
        // let this CTA's copies still in flight land (bounded)
        const int outstanding = issued < FS_STAGES ? issued : FS_STAGES;
        for (int i = 1; i <= outstanding; ++i) {
          int s = stage - i;
          uint32_t ph = phase;
          if (s < 0) { s += FS_STAGES; ph ^= 1u; }
          const long long t0 = clock64();
          while (!tc::mbar_try_wait(full + s, ph) && clock64() - t0 < tc::kWaitCycles) {}
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint32_t idS = tc::idesc_bf16(128, true);
      const uint32_t idA = tc::idesc_bf16(a.r2, true);
      const uint32_t idY = tc::idesc_bf16(256, true);
      const uint32_t sz = tc::smem_u32(smem + FS_Z_OFF);
      const uint32_t sh = tc::smem_u32(smem + FS_H_OFF);
      const uint32_t acc2 = tmem_base + 256u;
      // one k-block of 64 from the ring against a K-major A block at a_blk
      auto kblock = [&](uint32_t a_blk, uint32_t d, uint32_t idesc, bool first) -> bool {
        if (!tc::mbar_wait(full + stage, phase, abort_flag, a.status)) return false;
        tc::fence_after_sync();
        const uint32_t sb = tc::smem_u32(smem + FS_RING_OFF + stage * FS_SLOT);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t ad = tc::sdesc_sw128(a_blk + k * 32, 16, 1024);
          const uint64_t bd = tc::sdesc_sw128(sb + k * 2048, 8192, 1024);
          tc::mma_bf16(d, ad, bd, idesc, (first && k == 0) ? 0u : 1u);
        }
        tc::mma_commit(empty + stage);
        if (++stage == FS_STAGES) { stage = 0; phase ^= 1u; }
        return true;
      };
      int it = 0;
      long long v_done = 0;  // output passes issued so far (all tiles)
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++it) {
        if (!tc::mbar_wait(z_full, (uint32_t)it & 1u, abort_flag, a.status)) { ok = false; break; }
        tc::fence_after_sync();
        // the previous tile's last output pass must have been read out of
        // TMEM columns 0..255 before S overwrites them
        if (v_done > 0 && !tc::mbar_wait(y_empty, (uint32_t)((v_done - 1) & 1), abort_flag, a.status)) {
          ok = false;
          break;
        }
        for (int c = 0; c <= NC && ok; ++c) {
          if (c < NC) {
            const long long u = (long long)it * NC + c;
            const int b = (int)(u & 1);
            if (!tc::mbar_wait(s_empty + b, ((uint32_t)(u >> 1) & 1u) ^ 1u, abort_flag, a.status)) { ok = false; break; }
            tc::fence_after_sync();
            for (int kb = 0; kb < KB1 && ok; ++kb) ok = kblock(sz + kb * FS_BLK, tmem_base + b * 128u, idS, kb == 0);
            if (!ok) break;
            tc::mma_commit(s_full + b);
          }
          if (c >= 1) {  // acc2 += H[c-1] . U2[chunk c-1]
            const long long u = (long long)it * NC + c - 1;
            const int hb = (int)(u & 1);
            if (!tc::mbar_wait(h_full + hb, (uint32_t)(u >> 1) & 1u, abort_flag, a.status)) { ok = false; break; }
            tc::fence_after_sync();
            for (int kb = 0; kb < 2 && ok; ++kb)
              ok = kblock(sh + (hb * 2 + kb) * FS_BLK, acc2, idA, c == 1 && kb == 0);
            if (!ok) break;
            tc::mma_commit(h_empty + hb);
          }
        }
        if (!ok) break;
        tc::mma_commit(acc_full);
        // z2 replaces z1 in shared memory (written by the epilogue)
        if (!tc::mbar_wait(z2_full, (uint32_t)it & 1u, abort_flag, a.status)) { ok = false; break; }
        tc::fence_after_sync();
        for (int p = 0; p < NP && ok; ++p) {
          // TMEM columns 0..255: S of the last two chunks (p == 0) or the
          // previous pass must have been read out
          if (p == 0) {
            for (int j = 1; j <= 2 && j <= NC && ok; ++j) {
              const long long u = (long long)it * NC + NC - j;
              ok = tc::mbar_wait(s_empty + (int)(u & 1), (uint32_t)(u >> 1) & 1u, abort_flag, a.status);
            }
          } else {
            ok = tc::mbar_wait(y_empty, (uint32_t)((v_done - 1) & 1), abort_flag, a.status);
          }
          if (!ok) break;
          tc::fence_after_sync();
          for (int kb = 0; kb < KB2 && ok; ++kb) ok = kblock(sz + kb * FS_BLK, tmem_base, idY, kb == 0);
          if (!ok) break;
          tc::mma_commit(y_full);
          ++v_done;
        }
        if (ok) tc::mma_commit(z_empty);  // every MMA reading z2 is done once it fires
      }
      tc::mma_commit(drain);
      const long long t0 = clock64();
      while (!tc::mbar_try_wait(drain, 0) && clock64() - t0 < tc::kWaitCycles) {}
    }
  } else {
    // --------------------------------------------------------- epilogue --
    // Warp w reads TMEM lanes 32 (w % 4) .. + 31 (its 32 rows of the tile);
    // the four warps of a lane quadrant take a quarter of the columns each.
    const int q = warp & 3;
    const int part = (warp - 2) >> 2;   // 0 .. FS_NPART - 1
    const int row = q * 32 + lane;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    // tcgen05.ld is warp-collective: every wait result is made warp-uniform
    auto wwait = [&](uint64_t* bar, uint32_t par) {
      return __all_sync(0xffffffffu, tc::mbar_wait(bar, par, abort_flag, a.status)) != 0;
    };
    bool ok = true;
    int it = 0;
    long long v = 0;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++it) {
      const int m = t * 128 + row;
      const bool mok = m < a.M;
      for (int c = 0; c < NC && ok; ++c) {
        const long long u = (long long)it * NC + c;
        const int b = (int)(u & 1);
        const uint32_t k = (uint32_t)(u >> 1) & 1u;
        if (!wwait(s_full + b, k)) { ok = false; break; }
        tc::fence_after_sync();
        uint32_t r[FS_CPW];
        const uint32_t sc = tmem_base + lane_base + (uint32_t)(b * 128 + part * FS_CPW);
        tc::tmem_ld32(sc, r);
        tc::tmem_ld_wait();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(s_empty + b);  // S[b] may be overwritten now
        // + b1, GELU (columns past f: S = 0 from the zero-filled V1 and no
        // bias, so H = GELU(0) = 0 there)
        const int col0 = c * 128 + part * FS_CPW;
        float x[FS_CPW];
#pragma unroll
        for (int j = 0; j < FS_CPW; ++j) x[j] = __uint_as_float(r[j]);
        if (a.b1) {
          // 8 bias values per 16-byte load (f is a multiple of 8)
#pragma unroll
          for (int g8 = 0; g8 < FS_CPW / 8; ++g8) {
            const int col = col0 + 8 * g8;
            if (col < a.f) {
              const uint4 bb = __ldg(reinterpret_cast<const uint4*>(a.b1 + col));
              x[8 * g8 + 0] += bf_lo(bb.x); x[8 * g8 + 1] += bf_hi(bb.x);
              x[8 * g8 + 2] += bf_lo(bb.y); x[8 * g8 + 3] += bf_hi(bb.y);
              x[8 * g8 + 4] += bf_lo(bb.z); x[8 * g8 + 5] += bf_hi(bb.z);
              x[8 * g8 + 6] += bf_lo(bb.w); x[8 * g8 + 7] += bf_hi(bb.w);
            }
          }
        }
#pragma unroll
        for (int j = 0; j < FS_CPW; j += 2) gelu_erf2(x[j], x[j + 1]);
        // H[b] must have been consumed by the MMA of chunk u - 2
        if (!wwait(h_empty + b, k ^ 1u)) { ok = false; break; }
        // columns part * FS_CPW .. of the chunk: A block (col >> 6), 16-byte
        // chunks ((col & 63) >> 3) .. of the 128-byte swizzled row
        const int hc0 = part * FS_CPW;
        uint8_t* hblk = smem + FS_H_OFF + (b * 2 + (hc0 >> 6)) * FS_BLK;
#pragma unroll
        for (int ch = 0; ch < FS_CPW / 8; ++ch) {
          uint4 w;
          w.x = pack2(x[ch * 8 + 0], x[ch * 8 + 1]);
          w.y = pack2(x[ch * 8 + 2], x[ch * 8 + 3]);
          w.z = pack2(x[ch * 8 + 4], x[ch * 8 + 5]);
          w.w = pack2(x[ch * 8 + 6], x[ch * 8 + 7]);
          const int c16 = ((hc0 & 63) >> 3) + ch;
          *reinterpret_cast<uint4*>(hblk + row * 128 + ((c16 ^ (row & 7)) << 4)) = w;
        }
        tc::fence_proxy_async_smem();  // H is read by the tensor cores
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(h_full + b);
      }
      if (!ok) break;
      // ---- acc2 -> bf16 z2, over z1 in shared memory (every MMA that read
      // z1 has completed once acc_full fires) ----
      if (!wwait(acc_full, (uint32_t)it & 1u)) { ok = false; break; }
      tc::fence_after_sync();
      // 32-column groups g = part, part + FS_NPART, ... (r2 / 32 groups in all)
      for (int g = part; g < 2 * KB2; g += FS_NPART) {
        uint32_t r[32];
        tc::tmem_ld32(tmem_base + lane_base + 256u + (uint32_t)(32 * g), r);
        tc::tmem_ld_wait();
        const int col = 32 * g;                        // first of 32 columns
        uint8_t* zblk = smem + FS_Z_OFF + (col >> 6) * FS_BLK;
        const int ch0 = (col & 63) >> 3;                // 4 chunks of 8
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint4 w;
          w.x = pack2(__uint_as_float(r[cc * 8 + 0]), __uint_as_float(r[cc * 8 + 1]));
          w.y = pack2(__uint_as_float(r[cc * 8 + 2]), __uint_as_float(r[cc * 8 + 3]));
          w.z = pack2(__uint_as_float(r[cc * 8 + 4]), __uint_as_float(r[cc * 8 + 5]));
          w.w = pack2(__uint_as_float(r[cc * 8 + 6]), __uint_as_float(r[cc * 8 + 7]));
          *reinterpret_cast<uint4*>(zblk + row * 128 + (((ch0 + cc) ^ (row & 7)) << 4)) = w;
        }
      }
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(z2_full);
      if (a.discard && q == 0 && part == 0) {
        // every MMA that read this tile's z1 has completed (acc_full), and
        // no other tile reads these rows: drop their L2 lines without
        // write-back (whole 128-byte lines inside the tile's rows only)
        const int m0 = t * 128;
        const long long b0 = (long long)m0 * a.ldz * 2;
        const long long b1 = (long long)min(m0 + 128, a.M) * a.ldz * 2;
        const uintptr_t base = reinterpret_cast<uintptr_t>(a.z1);
        const uintptr_t l0 = (base + b0 + 127) & ~(uintptr_t)127, l1 = (base + b1) & ~(uintptr_t)127;
        for (uintptr_t ln = l0 + (uintptr_t)lane * 128; ln < l1; ln += 32 * 128)
          asm volatile("discard.global.L2 [%0], 128;" ::"l"(ln) : "memory");
      }
      // ---- output passes: y = z2 . V2 + b2 + resid ----
      for (int p = 0; p < NP && ok; ++p, ++v) {
        if (!wwait(y_full, (uint32_t)(v & 1))) { ok = false; break; }
        tc::fence_after_sync();
        for (int j = 0; j < 256 / (32 * FS_NPART); ++j) {
          uint32_t r[32];
          const int pc = part * (256 / FS_NPART) + 32 * j;   // column within the pass
          tc::tmem_ld32(tmem_base + lane_base + (uint32_t)pc, r);
          tc::tmem_ld_wait();
          const int col0 = p * 256 + pc;
          if (!mok) continue;
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            const int col = col0 + e;
            if (col >= a.d) break;  // d is a multiple of 8
            float o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = __uint_as_float(r[e + i]);
            if (a.b2) {
              const uint4 bb = __ldg(reinterpret_cast<const uint4*>(a.b2 + col));
              o[0] += bf_lo(bb.x); o[1] += bf_hi(bb.x); o[2] += bf_lo(bb.y); o[3] += bf_hi(bb.y);
              o[4] += bf_lo(bb.z); o[5] += bf_hi(bb.z); o[6] += bf_lo(bb.w); o[7] += bf_hi(bb.w);
            }
            if (a.resid) {
              const uint4 rr = *reinterpret_cast<const uint4*>(a.resid + (long long)m * a.d + col);
              o[0] += bf_lo(rr.x); o[1] += bf_hi(rr.x); o[2] += bf_lo(rr.y); o[3] += bf_hi(rr.y);
              o[4] += bf_lo(rr.z); o[5] += bf_hi(rr.z); o[6] += bf_lo(rr.w); o[7] += bf_hi(rr.w);
            }
            uint4 w;
            w.x = pack2(o[0], o[1]); w.y = pack2(o[2], o[3]); w.z = pack2(o[4], o[5]); w.w = pack2(o[6], o[7]);
            *reinterpret_cast<uint4*>(a.y + (long long)m * a.d + col) = w;
          }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(y_empty);
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem_base, FS_TMEM_COLS);
  }
}

}  // namespace

// z1 [M x r1] (row stride ldz), V1 [r1 x f], b1 [f] (or null), U2 [f x r2],
// V2 [r2 x d], b2 [d] (or null), resid [M x d] (or null, may alias y).
int ffn_stream_launch(const bf16* z1, long long ldz, const bf16* V1, const bf16* b1, const bf16* U2,
                      const bf16* V2, const bf16* b2, const bf16* resid, bf16* y, int M, int f, int r1,
                      int r2, int d, int* status, int sms, bool discard, cudaStream_t stream) {
  if (M <= 0 || f <= 0 || d <= 0) return FLASHSVD_ERR_INVALID_ARG;
  if (r1 % 64 || r2 % 64 || r1 < 64 || r2 < 64 || r1 > FS_RMAX || r2 > FS_RMAX || f % 8 || d % 8)
    return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  CUtensorMap mz, mv1, mu2, mv2;
  FSVD_TRY(encode_map(&mz, z1, M, r1, ldz, 64, 128, true));
  FSVD_TRY(encode_map(&mv1, V1, r1, f, f, 64, 64, true));
  FSVD_TRY(encode_map(&mu2, U2, f, r2, r2, 64, 64, true));
  FSVD_TRY(encode_map(&mv2, V2, r2, d, d, 64, 64, true));
  static SmemAttrOnce smem_once;
  FSVD_TRY(set_smem_once(smem_once, ffn_stream_kernel, FS_SMEM));
  FsArgs a;
  a.M = M; a.f = f; a.r1 = r1; a.r2 = r2; a.d = d;
  a.z1 = z1; a.ldz = ldz; a.discard = discard ? 1 : 0;
  a.b1 = b1; a.b2 = b2; a.resid = resid; a.y = y; a.status = status;
  const int tiles = (M + 127) / 128;
  const int grid = tiles < sms ? tiles : sms;
  const double flops = 2.0 * M * ((double)r1 * f + (double)f * r2 + (double)r2 * d);
  const double bytes = 2.0 * ((double)M * r1 + (double)r1 * f + (double)f * r2 + (double)r2 * d + 2.0 * M * d);
  const LaunchTag tag{"ffn_stream", bytes, flops};
  return launch_pdl(tag, ffn_stream_kernel, dim3(grid), dim3(FS_THREADS), (size_t)FS_SMEM, stream, mz, mv1, mu2,
                    mv2, a);
}

}  // namespace fsvd
