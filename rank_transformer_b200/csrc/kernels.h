// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace fsvd {

// ------------------------------------------------ decode split-K GEMV ----
// One launch computes, for up to three "problems" that share the same
// activation rows and the same reduction length K,
//     out[m, cols] = A[m, a_col + k] . W[k, cols]      (k < K)
// for rows m in [m0, m0+M), M <= 8, with the reduction split over CTAs and
// finished deterministically by the last CTA of each column tile.

enum GvPro { PRO_F32 = 0, PRO_BF16 = 1, PRO_RMSNORM = 2 };
enum GvEpi { EPI_F32 = 0, EPI_BF16 = 1, EPI_QKV = 2, EPI_SWIGLU = 3 };

struct GvProblem {
  const bf16* W;     // [K x N] (row stride ldw)
  long long ldw;
  long long w_row2;  // SWIGLU: first W row of the "up" half
  int a_col;         // first A column read
  int a_col2;        // SWIGLU: first A column of the "up" half
  int N;             // output columns
  int out_col;       // EPI_F32: column offset of this problem in out32
  int kind;          // EPI_QKV: 0 = q, 1 = k, 2 = v
};

struct GvParams {
  int M, m0, K, KC, splits, nprob;
  int tile_start[4];
  GvProblem prob[3];
  // A operand
  const float* a32; long long lda;                  // PRO_F32
  const bf16* x; long long ldx;                     // PRO_BF16 / PRO_RMSNORM
  const bf16* norm_g; float eps;                    // PRO_RMSNORM (row width K)
  // epilogue
  float* out32; long long ldo32;                    // EPI_F32
  bf16* out16; long long ldo16;                     // EPI_BF16 / QKV(q) / SWIGLU
  const bf16* bias;                                 // EPI_BF16 (may be null)
  const bf16* resid; long long ldr;                 // EPI_BF16 (may be null)
  bf16* k_cache; bf16* v_cache; const int* seqlens; // EPI_QKV
  int S_max, HD, D;
  const float* rope_cos; const float* rope_sin;     // [S_max x D/2]
  // workspace
  float* part; int* counters;
  long long part_cap; int counters_cap;             // their sizes (floats, ints)
};

enum GvMap { MAP_PLAIN = 0, MAP_ROPE = 1, MAP_SWIGLU = 2 };

// Host launcher: fills tile_start/splits/KC, picks the row-tile variant and
// launches once (row groups of up to 8 as the grid's third dimension).
int gemv_launch(GvParams p, int pro, int epi, int map, int total_rows,
                int target_ctas, cudaStream_t stream);
int gemv_tiles_for(int map, int N, int D);

// ---------------------------------------------- dense-KV decode attention --
struct AttnDecParams {
  const bf16* q; const bf16* k_new; const bf16* v_new;
  bf16* k_cache; bf16* v_cache; const int* seqlens; bf16* out;
  int B, H, D, S_max, nsplit, chunk;
  float scale_log2;              // scale * log2(e)
  float* part; int* counters;
};
int attn_decode_launch(AttnDecParams p, int target_ctas, cudaStream_t stream);

// ----------------------------------------------------------------- glue --
int rmsnorm_launch(const bf16* x, const bf16* g, bf16* y, int M, int d,
                   float eps, cudaStream_t s);
int layernorm_launch(const bf16* x, const bf16* g, const bf16* b, bf16* y,
                     int M, int d, float eps, cudaStream_t s);
int rope_table_launch(float* c, float* sn, int S_max, int D, float base,
                      cudaStream_t s);
int embed_launch(const int* tokens, const bf16* emb, bf16* x, int B, int d,
                 int vocab, cudaStream_t s);
int greedy_launch(const float* logits, int* next, int M, int vocab,
                  cudaStream_t s);
int advance_launch(int* seqlens, int B, cudaStream_t s);

// ------------------------------------------ prefill (tcgen05) linears ----
enum PfEpi { PF_EPI_BF16 = 0, PF_EPI_QKV = 1, PF_EPI_SWIGLU = 2, PF_EPI_GELU = 3,
             PF_EPI_F32 = 4 };

struct PfLinear {
  const bf16* x; long long ldx;      // A rows [M x d]
  const bf16* U; const bf16* V;      // [d x r], [r x n] (SWIGLU: V rows 0..r/2-1 gate, r/2.. up)
  const bf16* bias;                  // [n] or null
  const bf16* resid; long long ldr;  // [M x n] or null (added after bias/activation)
  bf16* y; long long ldy;            // output
  float* y32;                        // PF_EPI_F32 output (ld = ldy)
  int M, d, r, n;
  int epi;
  // QKV epilogue: y is the q buffer for kind 0; k/v rows go to the caches.
  int kind; bf16* cache; int S, S_max, HD, D;
  const float* rope_cos; const float* rope_sin;
  bf16* z;                           // [M x r] bf16 scratch for the rank activations
  int* zcnt;                         // [ceil(M / 128)] zero counters: z blocks discarded from L2 after use, or null
  int* status;
  int z_ready;                       // z already holds x . U (stage 1 skipped)
};
int prefill_linear_launch(const PfLinear& p, cudaStream_t stream);
// Stage 1 of n <= 3 factorized linears sharing x, in one tcgen05 launch:
// z[i] [M x r[i]] = x . U[i] (bf16, row stride r[i]).
int prefill_stage1_grouped(const bf16* x, long long ldx, int d, int M, int n, const bf16* const* U,
                           const int* r, bf16* const* z, int* status, cudaStream_t stream);
int prefill_dense_launch(const PfLinear& p, cudaStream_t stream);
// Stage 2 of n <= 3 of the q, k, v projections in one tcgen05 launch.  The
// rank activations are stacked in one buffer z (row stride r, equal ranks):
// problem i reads rows row[i] .. row[i] + M; kind[i] 0 = q (to q, row stride
// ldq), 1 = k, 2 = v (to cache[i] [B, S_max, H, D] rows 0..S-1, as the
// single-problem QKV epilogue); bias[i] may be null; RoPE on q and k when
// the tables are given.  zcnt (3 x ceil(M / 128) zero counters) or null:
// each problem's z rows are discarded from L2 after their last use.
struct QkvGroup {
  int n, M, r;
  const bf16* z; int row[3];
  const bf16* V[3]; const bf16* bias[3]; int kind[3];
  bf16* cache[3]; bf16* q; long long ldq;
  int S, S_max, HD, D;
  const float* rope_cos; const float* rope_sin;
  int* zcnt; int* status;
};
int prefill_qkv_stage2_grouped(const QkvGroup& g, cudaStream_t stream);
// Stage 1 of one factorized linear: z [M x r] (row stride r) = x . U, bf16.
int prefill_stage1(const bf16* x, long long ldx, int d, int M, const bf16* U, int r, bf16* z, int* status,
                   cudaStream_t stream);

// Streamed low-rank FFN (ffn_stream.cu): y = GELU(z1 . V1 + b1) . U2 . V2 + b2
// + resid with z1 = x . U1 given [M x r1] (row stride ldz); the [M x f]
// activation stays on chip.  r1, r2 multiples of 64 in [64, 256]; b1, b2,
// resid may be null; resid may alias y.
constexpr int kFfnStreamMaxRank = 256;
int ffn_stream_launch(const bf16* z1, long long ldz, const bf16* V1, const bf16* b1, const bf16* U2,
                      const bf16* V2, const bf16* b2, const bf16* resid, bf16* y, int M, int f, int r1,
                      int r2, int d, int* status, int sms, bool discard, cudaStream_t stream);

// --------------------------------------------- fused decode layer ---------
struct DecodeLayerDesc {
  const bf16 *U[3], *V[3], *U_o, *V_o, *U_gu, *V_gu, *U_dn, *V_dn;
  const bf16 *g1, *g2;
  int d, H, D, f, r, r_f;
  float eps;
  const float *rope_cos, *rope_sin;
  const void* pack;  // the layer's decode pack (decode_pack_launch), or null
};
int decode_fused_supported(int B, int d, int D, int r, int r_f);
long long decode_pack_bytes(const DecodeLayerDesc& L, int sm_count);
int decode_pack_launch(const DecodeLayerDesc& L, void* dst, long long bytes, int sm_count,
                       cudaStream_t stream);
// Fused decode layer; x is updated in place.  xm: [B x d] bf16 scratch;
// part: fp32 partial slots (>= 2 * sm_count * 16 * 640 floats); bar: 9 stage
// counters and done: 1 counter, all zero between launches.
int decode_fused_launch(const DecodeLayerDesc& L, bf16* x, bf16* kc, bf16* vc, const int* seqlens,
                        int B, int S_max, bf16* xm, float* part, long long part_floats, int* bar,
                        int* done, int* status, int sm_count, cudaStream_t stream);
// Several layers in one launch (layer i on caches k_caches[i], v_caches[i]);
// the plan owns a device copy of the layers' descriptors.
struct DecodePlan;
int decode_plan_create(const DecodeLayerDesc* layers, int n, bf16* const* k_caches, bf16* const* v_caches,
                       int B, int S_max, int sm_count, DecodePlan** out);
int decode_plan_launch(const DecodePlan* plan, bf16* x, const int* seqlens, bf16* xm, float* part,
                       long long part_floats, int* bar, int* done, int* status, cudaStream_t stream);
void decode_plan_destroy(DecodePlan* plan);
int encode_map(CUtensorMap* map, const void* base, long long rows, long long cols, long long ld,
               int box_cols, int box_rows, bool swizzle128);
constexpr int kFusedPartFloats = 2 * 148 * 16 * 640;
// Test hook (flashsvd_debug_drop_barrier_arrival): when set, the next fused
// decode launch takes it (resetting it) and its CTA 0 skips its first
// grid-barrier arrival, so that the other CTAs' bounded waits expire.
extern std::atomic<int> g_df_drop_arrival;  // two halves; per SM 16 slots of 640 floats

// ------------------------------------------------ prefill attention -------
struct AttnPfParams {
  const bf16* q; const bf16* k; const bf16* v; bf16* out;
  int B, S, H, D, S_max, causal;
  float scale_log2;
  int* status;       // device status word (bounded waits)
  // Factorized query (zq non-null; q unused): q = rope(z_q V_q) is formed in
  // the kernel from z_q [B*S x r] (row stride ldz) and V_q [r x H*D], with
  // the rotary tables [S x D/2] at positions 0..S-1; r a multiple of 64.
  // zcnt: zero counters (zcnt_cap of them) for discarding z_q from L2 after
  // use, or null.
  const bf16* zq; long long ldz; int r; const bf16* Vq;
  const float* rope_cos; const float* rope_sin;
  int* zcnt; long long zcnt_cap;
};
int attn_prefill_launch(const AttnPfParams& p, cudaStream_t stream);

}  // namespace fsvd
