// C ABI of libflashsvd: argument checks, workspace, dispatch to the decode
// (M <= 32) or prefill (tcgen05) kernels, layer composition and per-layer
// CUDA-graph capture/replay.
#include <cstring>
#include <mutex>
#include <vector>

#include "kernels.h"

namespace fsvd {

std::atomic<int64_t> g_launches{0};
int g_last_cuda_error = 0;

namespace {

constexpr int DECODE_MAX_ROWS = 32;
constexpr int kCountersN = 1 << 16;

struct Ctx {
  int device = -1;
  int max_tokens = 0, max_rank = 0, max_hidden = 0, max_ffn = 0;
  int sm_count = 148;
  float* z = nullptr;          size_t z_elems = 0;
  float* part = nullptr;       size_t part_elems = 0;
  int* counters = nullptr;
  float* apart = nullptr;      size_t apart_elems = 0;
  int* acounters = nullptr;
  int* status = nullptr;
  bf16* xn = nullptr;          // [rows x max_hidden]
  bf16* q = nullptr;           // [rows x max_hidden]
  bf16* att = nullptr;         // [rows x max_hidden]
  bf16* h = nullptr;           // [rows x max_ffn]
  bf16* zb = nullptr;          // [rows x 2*max_rank] prefill rank activations
  float* df_part = nullptr;    // fused decode: per-CTA partial slots
  int* df_cnt = nullptr;       // fused decode: tile counters, stage barriers, done counter
  int* zcnt = nullptr;         // prefill: per 128-row block counters of the z discard
  long long zcnt_elems = 0;
  int rows = 0;                // rows of the scratch above
};

// The default context (flashsvd_init / flashsvd_shutdown) and the context a
// host thread has bound with flashsvd_ctx_bind (none: the default).
Ctx g_default;
thread_local Ctx* t_ctx = nullptr;
std::mutex g_mu;

inline Ctx& cur() { return t_ctx ? *t_ctx : g_default; }

// Whether prefill kernels drop a rank activation's L2 lines after its last
// use (discard.global.L2: no write-back to HBM).  On by default.
bool g_l2_discard = true;

void free_ctx(Ctx& c) {
  void* ptrs[] = {c.z, c.part, c.counters, c.apart, c.acounters, c.status,
                  c.xn, c.q, c.att, c.h, c.zb, c.df_part, c.df_cnt, c.zcnt};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  c = Ctx();
}

// Allocate and clear a context's workspace on `device` (which must be
// current).  On failure nothing stays allocated.
int alloc_ctx(Ctx& c, int device, int max_tokens, int max_rank, int max_hidden, int max_ffn) {
  c = Ctx();
  c.device = device;
  c.max_tokens = max_tokens; c.max_rank = max_rank;
  c.max_hidden = max_hidden; c.max_ffn = max_ffn;
  cudaDeviceGetAttribute(&c.sm_count, cudaDevAttrMultiProcessorCount, device);
  c.rows = max_tokens > DECODE_MAX_ROWS ? max_tokens : DECODE_MAX_ROWS;
  const int wide = max_ffn > max_hidden ? max_ffn : max_hidden;
  c.z_elems = (size_t)DECODE_MAX_ROWS * 3 * (max_rank > wide / 2 ? max_rank : wide / 2) + 4096;
  c.part_elems = (size_t)16 << 20;
  c.apart_elems = (size_t)16 << 20;  // split-sequence partials of decode attention
  cudaError_t e = cudaSuccess;
#define FSVD_ALLOC(ptr, bytes) \
  if (e == cudaSuccess) e = cudaMalloc((void**)&(ptr), (bytes));
  FSVD_ALLOC(c.z, c.z_elems * sizeof(float));
  FSVD_ALLOC(c.part, c.part_elems * sizeof(float));
  FSVD_ALLOC(c.counters, kCountersN * sizeof(int));
  FSVD_ALLOC(c.apart, c.apart_elems * sizeof(float));
  FSVD_ALLOC(c.acounters, kCountersN * sizeof(int));
  FSVD_ALLOC(c.status, 64 * sizeof(int));
  FSVD_ALLOC(c.xn, (size_t)c.rows * max_hidden * sizeof(bf16));
  FSVD_ALLOC(c.q, (size_t)c.rows * max_hidden * sizeof(bf16));
  FSVD_ALLOC(c.att, (size_t)c.rows * max_hidden * sizeof(bf16));
  FSVD_ALLOC(c.h, (size_t)c.rows * max_ffn * sizeof(bf16));
  FSVD_ALLOC(c.zb, (size_t)c.rows * 3 * max_rank * sizeof(bf16));  // grouped q/k/v stage 1: 3 ranks
  FSVD_ALLOC(c.df_part, (size_t)kFusedPartFloats * sizeof(float));
  FSVD_ALLOC(c.df_cnt, (size_t)(4096 + 64) * sizeof(int));
  // (the factorized attention counts per batch row and query tile: at most
  // rows / 128 + batch rows of them)
  c.zcnt_elems = (long long)(c.rows / 128 + 1) + (c.rows < (1 << 16) ? c.rows : (1 << 16));
  FSVD_ALLOC(c.zcnt, (size_t)c.zcnt_elems * sizeof(int));
#undef FSVD_ALLOC
  if (e == cudaSuccess) e = cudaMemset(c.counters, 0, kCountersN * sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(c.acounters, 0, kCountersN * sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(c.status, 0, 64 * sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(c.df_cnt, 0, (4096 + 64) * sizeof(int));
  if (e == cudaSuccess) e = cudaMemset(c.zcnt, 0, (size_t)c.zcnt_elems * sizeof(int));
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    free_ctx(c);
    g_last_cuda_error = (int)e;
    return e == cudaErrorMemoryAllocation ? FLASHSVD_ERR_NO_MEMORY : FLASHSVD_ERR_CUDA;
  }
  return FLASHSVD_OK;
}

bool capturing(cudaStream_t s) {
  cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &st) != cudaSuccess) return false;
  return st != cudaStreamCaptureStatusNone;
}

int need_init() { return cur().device < 0 ? FLASHSVD_ERR_NOT_INITIALIZED : FLASHSVD_OK; }

inline const bf16* cb(const flashsvd_bf16* p) { return reinterpret_cast<const bf16*>(p); }

int check_ptr(const void* p) {
  if (!p) return FLASHSVD_ERR_INVALID_ARG;
  if (!aligned16(p)) return FLASHSVD_ERR_MISALIGNED;
  return FLASHSVD_OK;
}
int check_opt_ptr(const void* p) { return p ? check_ptr(p) : FLASHSVD_OK; }
int check_w8(int v) {
  if (v <= 0) return FLASHSVD_ERR_INVALID_ARG;
  return (v % 8) ? FLASHSVD_ERR_UNSUPPORTED_SHAPE : FLASHSVD_OK;
}

int target_ctas() { return cur().sm_count * 3; }

// Capacity guard for decode attention: one partial of D + 2 floats per
// (batch, head, 64-key chunk).
int attn_fits(int B, int H, int D, int S_max) {
  const size_t chunks = (size_t)ceil_div(S_max, 64);
  if (chunks > 1024 || (size_t)B * H > (size_t)kCountersN ||
      (size_t)B * H * chunks * (D + 2) > cur().apart_elems)
    return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  return FLASHSVD_OK;
}

GvParams gv_base() {
  GvParams p;
  memset(&p, 0, sizeof(p));
  p.part = cur().part;
  p.counters = cur().counters;
  p.part_cap = (long long)cur().part_elems;
  p.counters_cap = kCountersN;
  return p;
}

// Capacity guard for the split-K partials of one GEMV launch.
int gv_fits(int K, int tiles) {
  const long long splits_max = ((long long)target_ctas() / tiles) + ceil_div(K, 512) + 1;
  if (tiles > kCountersN) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  if ((long long)tiles * splits_max * 512 > (long long)cur().part_elems)
    return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  return FLASHSVD_OK;
}

// Stage 1 of a decode linear: z[:, off_i : off_i + N_i] = A . U_i.
int decode_stage1(int pro, const bf16* x, long long ldx, const bf16* norm_g,
                  float eps, const bf16* const* U, const int* N, int nprob,
                  int K, int M, cudaStream_t s) {
  GvParams p = gv_base();
  p.K = K;
  p.nprob = nprob;
  p.x = x; p.ldx = ldx; p.norm_g = norm_g; p.eps = eps;
  int off = 0, tiles = 0;
  for (int i = 0; i < nprob; ++i) {
    p.prob[i].W = U[i]; p.prob[i].ldw = N[i]; p.prob[i].N = N[i];
    p.prob[i].out_col = off; p.prob[i].a_col = 0;
    off += N[i];
    tiles += gemv_tiles_for(MAP_PLAIN, N[i], 64);
  }
  if ((size_t)M * off > cur().z_elems) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  FSVD_TRY(gv_fits(K, tiles));
  p.out32 = cur().z; p.ldo32 = off;
  return gemv_launch(p, pro, EPI_F32, MAP_PLAIN, M, target_ctas(), s);
}

int decode_linear(const bf16* x, const bf16* U, const bf16* V, const bf16* bias,
                  const bf16* resid, bf16* y, int M, int d, int r, int n,
                  const bf16* norm_g, float eps, cudaStream_t s) {
  const bf16* Us[1] = {U};
  const int Ns[1] = {r};
  FSVD_TRY(decode_stage1(norm_g ? PRO_RMSNORM : PRO_BF16, x, d, norm_g, eps, Us, Ns, 1, d, M, s));
  GvParams p = gv_base();
  p.K = r; p.nprob = 1;
  p.prob[0].W = V; p.prob[0].ldw = n; p.prob[0].N = n;
  p.a32 = cur().z; p.lda = r;
  p.out16 = y; p.ldo16 = n; p.bias = bias; p.resid = resid; p.ldr = n;
  FSVD_TRY(gv_fits(r, gemv_tiles_for(MAP_PLAIN, n, 64)));
  return gemv_launch(p, PRO_F32, EPI_BF16, MAP_PLAIN, M, target_ctas(), s);
}

// Decode gate|up: h = SiLU(z_g V_g) * (z_u V_u), z = A . U_gu.
int decode_gateup(const bf16* x, const bf16* U_gu, const bf16* V_gu, bf16* h,
                  int M, int d, int r_f, int f, const bf16* norm_g, float eps,
                  cudaStream_t s) {
  const bf16* Us[1] = {U_gu};
  const int Ns[1] = {2 * r_f};
  FSVD_TRY(decode_stage1(norm_g ? PRO_RMSNORM : PRO_BF16, x, d, norm_g, eps, Us, Ns, 1, d, M, s));
  GvParams p = gv_base();
  p.K = r_f; p.nprob = 1;
  p.prob[0].W = V_gu; p.prob[0].ldw = f; p.prob[0].N = f;
  p.prob[0].a_col = 0; p.prob[0].a_col2 = r_f; p.prob[0].w_row2 = r_f;
  p.a32 = cur().z; p.lda = 2 * r_f;
  p.out16 = h; p.ldo16 = f;
  FSVD_TRY(gv_fits(r_f, gemv_tiles_for(MAP_SWIGLU, f, 64)));
  return gemv_launch(p, PRO_F32, EPI_SWIGLU, MAP_SWIGLU, M, target_ctas(), s);
}

int ensure_scratch(int rows, int hidden, int ffn) {
  if (rows > cur().rows || hidden > cur().max_hidden || ffn > cur().max_ffn)
    return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  return FLASHSVD_OK;
}

int check_factor(const flashsvd_factor& F, int d_in, int d_out, bool bias_ok) {
  FSVD_TRY(check_ptr(F.U));
  FSVD_TRY(check_ptr(F.V));
  if (!bias_ok && F.bias) return FLASHSVD_ERR_INVALID_ARG;
  FSVD_TRY(check_opt_ptr(F.bias));
  FSVD_TRY(check_w8(F.r));
  if (F.r > cur().max_rank) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  (void)d_in; (void)d_out;
  return FLASHSVD_OK;
}

// Whether the streamed low-rank FFN kernel covers an encoder FFN of these
// shapes (d -> f at rank r1, f -> d at rank r2).
bool ffn_stream_covers(int d, int r1, int f, int r2) {
  return d % 64 == 0 && r1 % 64 == 0 && r2 % 64 == 0 && r1 >= 64 && r2 >= 64 &&
         r1 <= kFfnStreamMaxRank && r2 <= kFfnStreamMaxRank && f % 8 == 0;
}

int check_layer(const flashsvd_layer* L) {
  if (!L) return FLASHSVD_ERR_INVALID_ARG;
  if (L->kind != FLASHSVD_DECODER && L->kind != FLASHSVD_ENCODER) return FLASHSVD_ERR_INVALID_ARG;
  FSVD_TRY(check_w8(L->d));
  FSVD_TRY(check_w8(L->f));
  if (L->H <= 0 || L->D <= 0 || L->H * L->D != L->d) return FLASHSVD_ERR_INVALID_ARG;
  if (L->D != 64 && L->D != 128) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  const bool enc = L->kind == FLASHSVD_ENCODER;
  // a streamed encoder FFN keeps its [M x f] activation on chip: f is not
  // bounded by the workspace
  const bool streamed = enc && ffn_stream_covers(L->d, L->up.r, L->f, L->down.r);
  if (L->d > cur().max_hidden || (L->f > cur().max_ffn && !streamed)) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  FSVD_TRY(check_factor(L->q, L->d, L->d, enc));
  FSVD_TRY(check_factor(L->k, L->d, L->d, enc));
  FSVD_TRY(check_factor(L->v, L->d, L->d, enc));
  FSVD_TRY(check_factor(L->o, L->d, L->d, enc));
  FSVD_TRY(check_factor(L->down, L->f, L->d, enc));
  FSVD_TRY(check_ptr(L->norm1_g));
  FSVD_TRY(check_ptr(L->norm2_g));
  if (enc) {
    FSVD_TRY(check_ptr(L->norm1_b));
    FSVD_TRY(check_ptr(L->norm2_b));
    FSVD_TRY(check_factor(L->up, L->d, L->f, true));
  } else {
    FSVD_TRY(check_ptr(L->U_gu));
    FSVD_TRY(check_ptr(L->V_gu));
    FSVD_TRY(check_w8(L->r_f));
    if (2 * L->r_f > cur().max_rank * 2) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
    FSVD_TRY(check_ptr(L->rope_cos));
    FSVD_TRY(check_ptr(L->rope_sin));
  }
  return FLASHSVD_OK;
}

PfLinear pf_base(const bf16* x, long long ldx, const flashsvd_factor& F, int M,
                 int d, int n, bf16* y, long long ldy) {
  PfLinear p;
  memset(&p, 0, sizeof(p));
  p.x = x; p.ldx = ldx; p.U = cb(F.U); p.V = cb(F.V); p.bias = cb(F.bias);
  p.y = y; p.ldy = ldy; p.M = M; p.d = d; p.r = F.r; p.n = n;
  p.epi = PF_EPI_BF16;
  p.z = cur().zb;
  p.zcnt = g_l2_discard ? cur().zcnt : nullptr;
  p.status = cur().status;
  return p;
}

// Stage 1 of the q, k, v projections of x in one grouped tcgen05 launch,
// into three regions of the rank-activation scratch; false (nothing
// launched) when they do not fit it together.
bool qkv_stage1_grouped(const bf16* x, int d, int M, const flashsvd_factor* const* F, bf16** z,
                        cudaStream_t s, int* st) {
  const long long need = (long long)M * (F[0]->r + F[1]->r + F[2]->r);
  if (need > (long long)cur().rows * 3 * cur().max_rank) return false;
  const bf16* U[3];
  int r[3];
  long long off = 0;
  for (int i = 0; i < 3; ++i) {
    U[i] = cb(F[i]->U);
    r[i] = F[i]->r;
    z[i] = cur().zb + off;
    off += (long long)M * r[i];
    if (!aligned16(z[i]) || r[i] % 8) return false;
  }
  *st = prefill_stage1_grouped(x, d, d, M, 3, U, r, z, cur().status, s);
  return true;
}

// Stage 2 of the q, k, v projections (those of `first` .. 2) as one grouped
// tcgen05 launch over the rank activations that the grouped stage 1 left
// stacked in the scratch (equal ranks): q to the q buffer, k and v (k with
// RoPE when the tables are given) into the caches.
int qkv_stage2_grouped(const flashsvd_factor* const* F, bf16* const* z, int first, int M, int d, int D, int S,
                       int S_max, bf16* q_out, bf16* kc, bf16* vc, const float* cos_t, const float* sin_t,
                       cudaStream_t s) {
  QkvGroup g;
  memset(&g, 0, sizeof(g));
  bf16* dst[3] = {nullptr, kc, vc};
  for (int i = first; i < 3; ++i) {
    g.row[g.n] = (int)((z[i] - z[0]) / F[0]->r);
    g.V[g.n] = cb(F[i]->V); g.bias[g.n] = cb(F[i]->bias); g.kind[g.n] = i; g.cache[g.n] = dst[i];
    ++g.n;
  }
  g.M = M; g.r = F[0]->r; g.z = z[0];
  g.q = q_out; g.ldq = d;
  g.S = S; g.S_max = S_max; g.HD = d; g.D = D;
  g.rope_cos = cos_t; g.rope_sin = sin_t;
  g.zcnt = g_l2_discard ? cur().zcnt : nullptr;
  g.status = cur().status;
  return prefill_qkv_stage2_grouped(g, s);
}

bool g_fused_decode = true;
// Prefill attention of decoder layers: query formed inside the attention
// kernel (1) or from the dense q projection (0, the default: measured faster
// at every query rank from 128 to 1216 on the 7B-shaped layer).
int g_prefill_qf = 0;

// Whether the fused decode layer (and hence a decode pack) covers L's shapes.
bool pack_shapes_ok(const flashsvd_layer* L) {
  const int r = L->q.r;
  return L->k.r == r && L->v.r == r && L->down.r == L->r_f && L->f % 8 == 0 &&
         decode_fused_supported(1, L->d, L->D, r, L->r_f);
}

DecodeLayerDesc decode_desc(const flashsvd_layer* L) {
  DecodeLayerDesc D;
  memset(&D, 0, sizeof(D));
  D.U[0] = cb(L->q.U); D.U[1] = cb(L->k.U); D.U[2] = cb(L->v.U);
  D.V[0] = cb(L->q.V); D.V[1] = cb(L->k.V); D.V[2] = cb(L->v.V);
  D.U_o = cb(L->o.U); D.V_o = cb(L->o.V);
  D.U_gu = cb(L->U_gu); D.V_gu = cb(L->V_gu);
  D.U_dn = cb(L->down.U); D.V_dn = cb(L->down.V);
  D.g1 = cb(L->norm1_g); D.g2 = cb(L->norm2_g);
  D.d = L->d; D.H = L->H; D.D = L->D; D.f = L->f; D.r = L->q.r; D.r_f = L->r_f;
  D.eps = L->norm_eps; D.rope_cos = L->rope_cos; D.rope_sin = L->rope_sin;
  D.pack = L->decode_pack;
  return D;
}

// ------------------------------------------------------- layer: decode ----
int layer_decode(const flashsvd_layer* L, bf16* x, bf16* kc, bf16* vc,
                 const int* seqlens, int B, int S_max, cudaStream_t s) {
  const int d = L->d, r = L->q.r;
  const bool same_r = L->k.r == r && L->v.r == r;
  if (g_fused_decode && L->decode_pack && pack_shapes_ok(L) && cur().sm_count <= 148 &&
      decode_fused_supported(B, d, L->D, r, L->r_f)) {
    const DecodeLayerDesc D = decode_desc(L);
    const int st = decode_fused_launch(D, x, kc, vc, seqlens, B, S_max, cur().xn, cur().df_part,
                                       kFusedPartFloats, cur().df_cnt, cur().df_cnt + 32, cur().status,
                                       cur().sm_count, s);
    if (st != FLASHSVD_ERR_UNSUPPORTED_SHAPE) return st;
  }
  // 1) z_qkv = rmsnorm(x) . [U_q | U_k | U_v]
  if (!same_r) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  {
    const bf16* Us[3] = {(const bf16*)L->q.U, (const bf16*)L->k.U, (const bf16*)L->v.U};
    const int Ns[3] = {r, r, r};
    FSVD_TRY(decode_stage1(PRO_RMSNORM, x, d, (const bf16*)L->norm1_g, L->norm_eps, Us, Ns, 3, d, B, s));
  }
  // 2) q, k, v = z . V (RoPE on q, k; k, v appended at cache_seqlens[b])
  {
    GvParams p = gv_base();
    p.K = r; p.nprob = 3;
    const bf16* Vs[3] = {(const bf16*)L->q.V, (const bf16*)L->k.V, (const bf16*)L->v.V};
    for (int i = 0; i < 3; ++i) {
      p.prob[i].W = Vs[i]; p.prob[i].ldw = d; p.prob[i].N = d;
      p.prob[i].a_col = i * r; p.prob[i].kind = i;
    }
    p.a32 = cur().z; p.lda = 3 * r;
    p.out16 = cur().q; p.ldo16 = d;
    p.k_cache = kc; p.v_cache = vc; p.seqlens = seqlens; p.S_max = S_max;
    p.HD = d; p.D = L->D;
    p.rope_cos = L->rope_cos; p.rope_sin = L->rope_sin;
    FSVD_TRY(gemv_launch(p, PRO_F32, EPI_QKV, MAP_ROPE, B, target_ctas(), s));
  }
  // 3) dense-KV attention over 0..pos
  FSVD_TRY(attn_fits(B, L->H, L->D, S_max));
  {
    AttnDecParams a;
    memset(&a, 0, sizeof(a));
    a.q = cur().q; a.k_cache = kc; a.v_cache = vc; a.seqlens = seqlens; a.out = cur().att;
    a.B = B; a.H = L->H; a.D = L->D; a.S_max = S_max;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)L->D);
    a.part = cur().apart; a.counters = cur().acounters;
    FSVD_TRY(attn_decode_launch(a, target_ctas(), s));
  }
  // 4-5) x = x + (att . U_o) . V_o
  FSVD_TRY(decode_linear(cur().att, cb(L->o.U), cb(L->o.V), nullptr, x, x, B, d, L->o.r, d, nullptr, 0.f, s));
  // 6-7) h = SiLU(gate) * up of rmsnorm(x)
  FSVD_TRY(decode_gateup(x, cb(L->U_gu), cb(L->V_gu), cur().h, B, d, L->r_f, L->f,
                         (const bf16*)L->norm2_g, L->norm_eps, s));
  // 8-9) x = x + (h . U_dn) . V_dn
  return decode_linear(cur().h, cb(L->down.U), cb(L->down.V), nullptr, x, x, B, L->f, L->down.r, d, nullptr, 0.f, s);
}

// ------------------------------------------------------ layer: prefill ----
int layer_prefill(const flashsvd_layer* L, bf16* x, bf16* kc, bf16* vc,
                  int B, int S, int S_max, cudaStream_t s) {
  const int d = L->d, M = B * S;
  FSVD_TRY(rmsnorm_launch(x, cb(L->norm1_g), cur().xn, M, d, L->norm_eps, s));
  const flashsvd_factor* F[3] = {&L->q, &L->k, &L->v};
  bf16* dst[3] = {cur().q, kc, vc};
  bf16* zg[3];
  int gst = FLASHSVD_OK;
  const bool grouped = qkv_stage1_grouped(cur().xn, d, M, F, zg, s, &gst);
  FSVD_TRY(gst);
  // Factorized attention ([v1.5] Methodology 2, "Prefill"): with z_q kept
  // from the grouped stage 1, the attention kernel forms q = rope(z_q V_q)
  // itself, so q's stage 2 is not run and dense q is never materialised.
  // k and v still go through stage 2: decode reads them from the cache.
  const bool fact_q = grouped && L->q.r % 64 == 0 && g_prefill_qf == 1;
  if (grouped && L->k.r == L->q.r && L->v.r == L->q.r) {
    FSVD_TRY(qkv_stage2_grouped(F, zg, fact_q ? 1 : 0, M, d, L->D, S, S_max, cur().q, kc, vc, L->rope_cos,
                                L->rope_sin, s));
  } else {
    for (int i = fact_q ? 1 : 0; i < 3; ++i) {
      PfLinear p = pf_base(cur().xn, d, *F[i], M, d, d, cur().q, d);
      if (grouped) { p.z = zg[i]; p.z_ready = 1; }
      p.epi = PF_EPI_QKV; p.kind = i; p.cache = dst[i]; p.S = S; p.S_max = S_max;
      p.HD = d; p.D = L->D;
      if (i < 2) { p.rope_cos = L->rope_cos; p.rope_sin = L->rope_sin; }
      FSVD_TRY(prefill_linear_launch(p, s));
    }
  }
  AttnPfParams a;
  memset(&a, 0, sizeof(a));
  a.k = kc; a.v = vc; a.out = cur().att;
  a.B = B; a.S = S; a.H = L->H; a.D = L->D; a.S_max = S_max; a.causal = 1;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)L->D);
  a.status = cur().status;
  if (fact_q) {
    a.zq = zg[0]; a.ldz = L->q.r; a.r = L->q.r; a.Vq = cb(L->q.V);
    a.rope_cos = L->rope_cos; a.rope_sin = L->rope_sin;
    a.zcnt = g_l2_discard ? cur().zcnt : nullptr; a.zcnt_cap = cur().zcnt_elems;
  } else {
    a.q = cur().q;
  }
  FSVD_TRY(attn_prefill_launch(a, s));
  {
    PfLinear p = pf_base(cur().att, d, L->o, M, d, d, x, d);
    p.resid = x; p.ldr = d;
    FSVD_TRY(prefill_linear_launch(p, s));
  }
  FSVD_TRY(rmsnorm_launch(x, cb(L->norm2_g), cur().xn, M, d, L->norm_eps, s));
  {
    flashsvd_factor gu = {L->U_gu, L->V_gu, nullptr, 2 * L->r_f};
    PfLinear p = pf_base(cur().xn, d, gu, M, d, L->f, cur().h, L->f);
    p.epi = PF_EPI_SWIGLU;
    FSVD_TRY(prefill_linear_launch(p, s));
  }
  PfLinear p = pf_base(cur().h, L->f, L->down, M, L->f, d, x, d);
  p.resid = x; p.ldr = d;
  return prefill_linear_launch(p, s);
}

// Streamed low-rank FFN: z1 = x . U1 (tcgen05 stage 1 into the rank
// scratch), then y = GELU(z1 . V1 + b1) . U2 . V2 + b2 + resid in one
// kernel that keeps the [M x f] activation on chip.
int lowrank_ffn(const bf16* x, const bf16* U1, const bf16* V1, const bf16* b1, const bf16* U2,
                const bf16* V2, const bf16* b2, const bf16* resid, bf16* y, int M, int d, int r1, int f,
                int r2, cudaStream_t s) {
  bf16* z = cur().zb;
  FSVD_TRY(prefill_stage1(x, d, d, M, U1, r1, z, cur().status, s));
  return ffn_stream_launch(z, r1, V1, b1, U2, V2, b2, resid, y, M, f, r1, r2, d, cur().status,
                           cur().sm_count, g_l2_discard, s);
}

// ------------------------------------------------------ layer: encoder ----
int layer_encoder(const flashsvd_layer* L, bf16* x, bf16* kc, bf16* vc,
                  int B, int S, int S_max, cudaStream_t s) {
  const int d = L->d, M = B * S;
  const flashsvd_factor* F[3] = {&L->q, &L->k, &L->v};
  bf16* dst[3] = {cur().q, kc, vc};
  bf16* zg[3];
  int gst = FLASHSVD_OK;
  const bool grouped = qkv_stage1_grouped(x, d, M, F, zg, s, &gst);
  FSVD_TRY(gst);
  if (grouped && L->k.r == L->q.r && L->v.r == L->q.r) {
    FSVD_TRY(qkv_stage2_grouped(F, zg, 0, M, d, L->D, S, S_max, cur().q, kc, vc, nullptr, nullptr, s));
  } else {
    for (int i = 0; i < 3; ++i) {
      PfLinear p = pf_base(x, d, *F[i], M, d, d, cur().q, d);
      if (grouped) { p.z = zg[i]; p.z_ready = 1; }
      p.epi = PF_EPI_QKV; p.kind = i; p.cache = dst[i]; p.S = S; p.S_max = S_max;
      p.HD = d; p.D = L->D;
      FSVD_TRY(prefill_linear_launch(p, s));
    }
  }
  AttnPfParams a;
  memset(&a, 0, sizeof(a));
  a.q = cur().q; a.k = kc; a.v = vc; a.out = cur().att;
  a.B = B; a.S = S; a.H = L->H; a.D = L->D; a.S_max = S_max; a.causal = 0;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)L->D);
  a.status = cur().status;
  FSVD_TRY(attn_prefill_launch(a, s));
  {
    PfLinear p = pf_base(cur().att, d, L->o, M, d, d, cur().xn, d);
    p.resid = x; p.ldr = d;
    FSVD_TRY(prefill_linear_launch(p, s));
  }
  FSVD_TRY(layernorm_launch(cur().xn, cb(L->norm1_g), cb(L->norm1_b), x, M, d, L->norm_eps, s));
  if (ffn_stream_covers(d, L->up.r, L->f, L->down.r)) {
    // the FFN streamed over f-tiles: GELU(up(x)) never leaves the SM
    FSVD_TRY(lowrank_ffn(x, cb(L->up.U), cb(L->up.V), cb(L->up.bias), cb(L->down.U), cb(L->down.V),
                         cb(L->down.bias), x, cur().xn, M, d, L->up.r, L->f, L->down.r, s));
  } else {
    {
      PfLinear p = pf_base(x, d, L->up, M, d, L->f, cur().h, L->f);
      p.epi = PF_EPI_GELU;
      FSVD_TRY(prefill_linear_launch(p, s));
    }
    PfLinear p = pf_base(cur().h, L->f, L->down, M, L->f, d, cur().xn, d);
    p.resid = x; p.ldr = d;
    FSVD_TRY(prefill_linear_launch(p, s));
  }
  return layernorm_launch(cur().xn, cb(L->norm2_g), cb(L->norm2_b), x, M, d, L->norm_eps, s);
}

}  // namespace
}  // namespace fsvd

struct flashsvd_graph {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  int kernels = 0;
};

using namespace fsvd;

namespace {

int count_kernels(cudaGraph_t g, int* out) {
  size_t n = 0;
  FSVD_CUDA(cudaGraphGetNodes(g, nullptr, &n));
  std::vector<cudaGraphNode_t> nodes(n);
  if (n) FSVD_CUDA(cudaGraphGetNodes(g, nodes.data(), &n));
  int k = 0;
  for (size_t i = 0; i < n; ++i) {
    cudaGraphNodeType t;
    FSVD_CUDA(cudaGraphNodeGetType(nodes[i], &t));
    if (t == cudaGraphNodeTypeKernel) {
      ++k;
    } else if (t == cudaGraphNodeTypeGraph) {
      cudaGraph_t child;
      FSVD_CUDA(cudaGraphChildGraphNodeGetGraph(nodes[i], &child));
      int kc = 0;
      FSVD_TRY(count_kernels(child, &kc));
      k += kc;
    }
  }
  *out = k;
  return FLASHSVD_OK;
}

int finish_graph(cudaGraph_t graph, flashsvd_graph** out) {
  flashsvd_graph* g = new flashsvd_graph();
  g->graph = graph;
  int st = count_kernels(graph, &g->kernels);
  if (st == FLASHSVD_OK) st = cuda_status(cudaGraphInstantiate(&g->exec, graph, 0));
  if (st != FLASHSVD_OK) {
    cudaGraphDestroy(graph);
    delete g;
    return st;
  }
  *out = g;
  return FLASHSVD_OK;
}

}  // namespace

extern "C" {

const char* flashsvd_status_string(int status) {
  switch (status) {
    case FLASHSVD_OK: return "ok";
    case FLASHSVD_ERR_INVALID_ARG: return "invalid argument";
    case FLASHSVD_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case FLASHSVD_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case FLASHSVD_ERR_NOT_INITIALIZED: return "flashsvd_init not called";
    case FLASHSVD_ERR_CAPTURE_UNSAFE: return "not allowed during stream capture";
    case FLASHSVD_ERR_CUDA: return "CUDA error";
    case FLASHSVD_ERR_TIMEOUT: return "device wait timed out";
    case FLASHSVD_ERR_NO_MEMORY: return "out of device memory";
    default: return "unknown status";
  }
}

int flashsvd_last_cuda_error(void) { return g_last_cuda_error; }
int flashsvd_version(void) { return 100; }

int flashsvd_debug_drop_barrier_arrival(void) {
  g_df_drop_arrival.store(1);
  return FLASHSVD_OK;
}

int flashsvd_set_l2_discard(int on) {
  g_l2_discard = on != 0;
  return FLASHSVD_OK;
}

int flashsvd_set_prefill_attention(int mode) {
  if (mode < 0 || mode > 1) return FLASHSVD_ERR_INVALID_ARG;
  g_prefill_qf = mode;
  return FLASHSVD_OK;
}

int flashsvd_set_decode_path(int fused) {
  g_fused_decode = fused != 0;
  return FLASHSVD_OK;
}
int64_t flashsvd_launch_count(void) { return g_launches.load(); }

int flashsvd_decode_pack_bytes(const flashsvd_layer* L, size_t* bytes) {
  if (!L || !bytes) return FLASHSVD_ERR_INVALID_ARG;
  if (L->kind != FLASHSVD_DECODER) return FLASHSVD_ERR_INVALID_ARG;
  if (!pack_shapes_ok(L)) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  int sms = 148, dev = 0;
  FSVD_CUDA(cudaGetDevice(&dev));
  FSVD_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  *bytes = (size_t)decode_pack_bytes(decode_desc(L), sms);
  return FLASHSVD_OK;
}

int flashsvd_decode_pack(const flashsvd_layer* L, void* dst, size_t bytes, flashsvd_stream stream) {
  size_t need = 0;
  FSVD_TRY(flashsvd_decode_pack_bytes(L, &need));
  if (!dst || bytes < need) return FLASHSVD_ERR_INVALID_ARG;
  if (!aligned16(dst)) return FLASHSVD_ERR_MISALIGNED;
  if (capturing((cudaStream_t)stream)) return FLASHSVD_ERR_CAPTURE_UNSAFE;
  const flashsvd_bf16* ptrs[] = {L->q.U, L->k.U, L->v.U, L->q.V, L->k.V, L->v.V, L->o.U, L->o.V,
                                 L->U_gu, L->V_gu, L->down.U, L->down.V};
  for (const flashsvd_bf16* q : ptrs) {
    if (!q) return FLASHSVD_ERR_INVALID_ARG;
    if (!aligned16(q)) return FLASHSVD_ERR_MISALIGNED;
  }
  int sms = 148, dev = 0;
  FSVD_CUDA(cudaGetDevice(&dev));
  FSVD_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  return decode_pack_launch(decode_desc(L), dst, (long long)bytes, sms, (cudaStream_t)stream);
}

struct flashsvd_decode_plan {
  DecodePlan* impl = nullptr;
  int device = -1, B = 0, d = 0;
};

int flashsvd_decode_plan_create(const flashsvd_layer* layers, int n_layers, flashsvd_bf16* const* k_caches,
                                flashsvd_bf16* const* v_caches, int B, int S_max,
                                flashsvd_decode_plan** plan) {
  FSVD_TRY(need_init());
  if (!layers || n_layers <= 0 || !k_caches || !v_caches || !plan || B <= 0 || S_max <= 0)
    return FLASHSVD_ERR_INVALID_ARG;
  if (capturing(nullptr)) return FLASHSVD_ERR_CAPTURE_UNSAFE;
  if (!g_fused_decode || cur().sm_count > 148) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  std::vector<DecodeLayerDesc> descs((size_t)n_layers);
  std::vector<bf16*> kc((size_t)n_layers), vc((size_t)n_layers);
  for (int i = 0; i < n_layers; ++i) {
    const flashsvd_layer* L = layers + i;
    if (L->kind != FLASHSVD_DECODER) return FLASHSVD_ERR_INVALID_ARG;
    if (!L->decode_pack || !pack_shapes_ok(L)) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
    if (!k_caches[i] || !v_caches[i]) return FLASHSVD_ERR_INVALID_ARG;
    if (!aligned16(k_caches[i]) || !aligned16(v_caches[i])) return FLASHSVD_ERR_MISALIGNED;
    descs[i] = decode_desc(L);
    kc[i] = reinterpret_cast<bf16*>(k_caches[i]);
    vc[i] = reinterpret_cast<bf16*>(v_caches[i]);
  }
  DecodePlan* impl = nullptr;
  FSVD_TRY(decode_plan_create(descs.data(), n_layers, kc.data(), vc.data(), B, S_max, cur().sm_count, &impl));
  flashsvd_decode_plan* out = new flashsvd_decode_plan();
  out->impl = impl;
  out->device = cur().device;
  out->B = B;
  out->d = layers[0].d;
  *plan = out;
  return FLASHSVD_OK;
}

int flashsvd_decode_plan_forward(const flashsvd_decode_plan* plan, flashsvd_bf16* x_inout,
                                 const int32_t* cache_seqlens, flashsvd_stream stream) {
  FSVD_TRY(need_init());
  if (!plan || !x_inout || !cache_seqlens) return FLASHSVD_ERR_INVALID_ARG;
  if (plan->device != cur().device) return FLASHSVD_ERR_INVALID_ARG;
  if (!aligned16(x_inout)) return FLASHSVD_ERR_MISALIGNED;
  if (plan->d > cur().max_hidden) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  return decode_plan_launch(plan->impl, reinterpret_cast<bf16*>(x_inout), cache_seqlens, cur().xn, cur().df_part,
                            kFusedPartFloats, cur().df_cnt, cur().df_cnt + 32, cur().status,
                            (cudaStream_t)stream);
}

int flashsvd_decode_plan_destroy(flashsvd_decode_plan* plan) {
  if (!plan) return FLASHSVD_OK;
  decode_plan_destroy(plan->impl);
  delete plan;
  return FLASHSVD_OK;
}

int flashsvd_init(int device, int max_tokens, int max_rank, int max_hidden,
                  int max_ffn) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (device < 0 || max_tokens <= 0 || max_rank <= 0 || max_hidden <= 0 || max_ffn <= 0)
    return FLASHSVD_ERR_INVALID_ARG;
  if (capturing(nullptr)) return FLASHSVD_ERR_CAPTURE_UNSAFE;
  Ctx& d = g_default;
  if (d.device == device && max_tokens <= d.max_tokens && max_rank <= d.max_rank &&
      max_hidden <= d.max_hidden && max_ffn <= d.max_ffn)
    return FLASHSVD_OK;
  FSVD_CUDA(cudaSetDevice(device));
  if (d.device >= 0) {
    cudaDeviceSynchronize();
    free_ctx(d);
  }
  Ctx c;
  FSVD_TRY(alloc_ctx(c, device, max_tokens, max_rank, max_hidden, max_ffn));
  d = c;
  return FLASHSVD_OK;
}

int flashsvd_shutdown(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_default.device < 0) return FLASHSVD_OK;
  cudaSetDevice(g_default.device);
  cudaDeviceSynchronize();
  free_ctx(g_default);
  return FLASHSVD_OK;
}

struct flashsvd_ctx {
  Ctx c;
};

int flashsvd_ctx_create(int device, int max_tokens, int max_rank, int max_hidden, int max_ffn,
                        flashsvd_ctx** ctx) {
  if (!ctx || device < 0 || max_tokens <= 0 || max_rank <= 0 || max_hidden <= 0 || max_ffn <= 0)
    return FLASHSVD_ERR_INVALID_ARG;
  if (capturing(nullptr)) return FLASHSVD_ERR_CAPTURE_UNSAFE;
  int prev = -1;
  FSVD_CUDA(cudaGetDevice(&prev));
  FSVD_CUDA(cudaSetDevice(device));
  Ctx c;
  const int st = alloc_ctx(c, device, max_tokens, max_rank, max_hidden, max_ffn);
  cudaSetDevice(prev);
  if (st != FLASHSVD_OK) return st;
  flashsvd_ctx* out = new flashsvd_ctx();
  out->c = c;
  *ctx = out;
  return FLASHSVD_OK;
}

int flashsvd_ctx_destroy(flashsvd_ctx* ctx) {
  if (!ctx) return FLASHSVD_ERR_INVALID_ARG;
  if (t_ctx == &ctx->c) t_ctx = nullptr;
  int prev = -1;
  cudaGetDevice(&prev);
  cudaSetDevice(ctx->c.device);
  cudaDeviceSynchronize();
  free_ctx(ctx->c);
  if (prev >= 0) cudaSetDevice(prev);
  delete ctx;
  return FLASHSVD_OK;
}

int flashsvd_ctx_bind(flashsvd_ctx* ctx) {
  if (ctx) FSVD_CUDA(cudaSetDevice(ctx->c.device));
  t_ctx = ctx ? &ctx->c : nullptr;
  return FLASHSVD_OK;
}

int flashsvd_check_device_status(flashsvd_stream stream) {
  FSVD_TRY(need_init());
  if (capturing(stream)) return FLASHSVD_ERR_CAPTURE_UNSAFE;
  FSVD_CUDA(cudaStreamSynchronize(stream));
  int word = 0;
  FSVD_CUDA(cudaMemcpy(&word, cur().status, sizeof(int), cudaMemcpyDeviceToHost));
  if (word != DEV_STATUS_OK) {
    FSVD_CUDA(cudaMemset(cur().status, 0, sizeof(int)));
    FSVD_CUDA(cudaMemset(cur().df_cnt, 0, (4096 + 64) * sizeof(int)));
    FSVD_CUDA(cudaMemset(cur().counters, 0, kCountersN * sizeof(int)));
    FSVD_CUDA(cudaMemset(cur().acounters, 0, kCountersN * sizeof(int)));
    FSVD_CUDA(cudaMemset(cur().zcnt, 0, (size_t)cur().zcnt_elems * sizeof(int)));
    return word == DEV_STATUS_SCHEDULE ? FLASHSVD_ERR_UNSUPPORTED_SHAPE : FLASHSVD_ERR_TIMEOUT;
  }
  return FLASHSVD_OK;
}

int flashsvd_lowrank_linear(const flashsvd_bf16* x, const flashsvd_bf16* U,
                            const flashsvd_bf16* V, const flashsvd_bf16* bias,
                            flashsvd_bf16* y, int M, int d, int r, int n,
                            flashsvd_stream stream) {
  FSVD_TRY(need_init());
  FSVD_TRY(check_ptr(x)); FSVD_TRY(check_ptr(U)); FSVD_TRY(check_ptr(V));
  FSVD_TRY(check_ptr(y)); FSVD_TRY(check_opt_ptr(bias));
  if (M < 0) return FLASHSVD_ERR_INVALID_ARG;
  FSVD_TRY(check_w8(d)); FSVD_TRY(check_w8(r)); FSVD_TRY(check_w8(n));
  if (M == 0) return FLASHSVD_OK;
  if (M > cur().rows || r > cur().max_rank) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  if (M <= DECODE_MAX_ROWS)
    return decode_linear((const bf16*)x, (const bf16*)U, (const bf16*)V, (const bf16*)bias,
                         nullptr, (bf16*)y, M, d, r, n, nullptr, 0.f, stream);
  flashsvd_factor F = {U, V, bias, r};
  PfLinear p = pf_base((const bf16*)x, d, F, M, d, n, (bf16*)y, n);
  return prefill_linear_launch(p, stream);
}

int flashsvd_dense_linear_f32(const flashsvd_bf16* x, const flashsvd_bf16* W,
                              float* y, int M, int d, int n,
                              flashsvd_stream stream) {
  FSVD_TRY(need_init());
  FSVD_TRY(check_ptr(x)); FSVD_TRY(check_ptr(W)); FSVD_TRY(check_ptr(y));
  if (M < 0) return FLASHSVD_ERR_INVALID_ARG;
  FSVD_TRY(check_w8(d)); FSVD_TRY(check_w8(n));
  if (M == 0) return FLASHSVD_OK;
  if (M > cur().rows) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  if (M <= DECODE_MAX_ROWS) {
    GvParams p = gv_base();
    p.K = d; p.nprob = 1;
    p.prob[0].W = (const bf16*)W; p.prob[0].ldw = n; p.prob[0].N = n;
    p.x = (const bf16*)x; p.ldx = d;
    p.out32 = y; p.ldo32 = n;
    FSVD_TRY(gv_fits(d, gemv_tiles_for(MAP_PLAIN, n, 64)));
    return gemv_launch(p, PRO_BF16, EPI_F32, MAP_PLAIN, M, target_ctas(), stream);
  }
  PfLinear p;
  memset(&p, 0, sizeof(p));
  p.x = (const bf16*)x; p.ldx = d; p.V = (const bf16*)W; p.y32 = y; p.ldy = n;
  p.M = M; p.d = d; p.r = d; p.n = n; p.epi = PF_EPI_F32; p.status = cur().status;
  return prefill_dense_launch(p, stream);
}

int flashsvd_head_logits(const flashsvd_bf16* x, const flashsvd_bf16* g, float eps,
                         const flashsvd_bf16* W, float* logits, int M, int d, int n,
                         flashsvd_stream stream) {
  FSVD_TRY(need_init());
  FSVD_TRY(check_ptr(x)); FSVD_TRY(check_opt_ptr(g)); FSVD_TRY(check_ptr(W));
  FSVD_TRY(check_ptr(logits));
  if (M < 0 || (g && !(eps >= 0.f))) return FLASHSVD_ERR_INVALID_ARG;
  FSVD_TRY(check_w8(d)); FSVD_TRY(check_w8(n));
  if (M == 0) return FLASHSVD_OK;
  if (M > DECODE_MAX_ROWS || M > cur().rows) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  GvParams p = gv_base();
  p.K = d; p.nprob = 1;
  p.prob[0].W = (const bf16*)W; p.prob[0].ldw = n; p.prob[0].N = n;
  p.x = (const bf16*)x; p.ldx = d;
  p.norm_g = (const bf16*)g; p.eps = eps;
  p.out32 = logits; p.ldo32 = n;
  FSVD_TRY(gv_fits(d, gemv_tiles_for(MAP_PLAIN, n, 64)));
  return gemv_launch(p, g ? PRO_RMSNORM : PRO_BF16, EPI_F32, MAP_PLAIN, M, target_ctas(), stream);
}

int flashsvd_gateup_swiglu(const flashsvd_bf16* x, const flashsvd_bf16* U_gu,
                           const flashsvd_bf16* V_gu, flashsvd_bf16* h, int M,
                           int d, int r_f, int f, flashsvd_stream stream) {
  FSVD_TRY(need_init());
  FSVD_TRY(check_ptr(x)); FSVD_TRY(check_ptr(U_gu)); FSVD_TRY(check_ptr(V_gu));
  FSVD_TRY(check_ptr(h));
  if (M < 0) return FLASHSVD_ERR_INVALID_ARG;
  FSVD_TRY(check_w8(d)); FSVD_TRY(check_w8(r_f)); FSVD_TRY(check_w8(f));
  if (M == 0) return FLASHSVD_OK;
  if (M > cur().rows || r_f > cur().max_rank) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  if (M <= DECODE_MAX_ROWS)
    return decode_gateup((const bf16*)x, (const bf16*)U_gu, (const bf16*)V_gu, (bf16*)h, M, d, r_f, f,
                         nullptr, 0.f, stream);
  flashsvd_factor gu = {U_gu, V_gu, nullptr, 2 * r_f};
  PfLinear p = pf_base((const bf16*)x, d, gu, M, d, f, (bf16*)h, f);
  p.epi = PF_EPI_SWIGLU;
  return prefill_linear_launch(p, stream);
}

int flashsvd_packed_gateup_mlp(const flashsvd_bf16* x,
                               const flashsvd_bf16* U_gu,
                               const flashsvd_bf16* V_gu,
                               const flashsvd_bf16* U_dn,
                               const flashsvd_bf16* V_dn, flashsvd_bf16* y,
                               int M, int d, int r_f, int f, int r_dn,
                               flashsvd_stream stream) {
  FSVD_TRY(need_init());
  FSVD_TRY(check_ptr(U_dn)); FSVD_TRY(check_ptr(V_dn)); FSVD_TRY(check_ptr(y));
  FSVD_TRY(check_w8(r_dn));
  if (M > 0 && (M > cur().rows || f > cur().max_ffn || r_dn > cur().max_rank))
    return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  FSVD_TRY(flashsvd_gateup_swiglu(x, U_gu, V_gu, (flashsvd_bf16*)cur().h, M, d, r_f, f, stream));
  if (M == 0) return FLASHSVD_OK;
  if (M <= DECODE_MAX_ROWS)
    return decode_linear(cur().h, (const bf16*)U_dn, (const bf16*)V_dn, nullptr, nullptr, (bf16*)y,
                         M, f, r_dn, d, nullptr, 0.f, stream);
  flashsvd_factor dn = {U_dn, V_dn, nullptr, r_dn};
  PfLinear p = pf_base(cur().h, f, dn, M, f, d, (bf16*)y, d);
  return prefill_linear_launch(p, stream);
}

int flashsvd_lowrank_ffn(const flashsvd_bf16* x, const flashsvd_bf16* U_up, const flashsvd_bf16* V_up,
                         const flashsvd_bf16* b_up, const flashsvd_bf16* U_dn, const flashsvd_bf16* V_dn,
                         const flashsvd_bf16* b_dn, const flashsvd_bf16* resid, flashsvd_bf16* y, int M,
                         int d, int r_up, int f, int r_dn, flashsvd_stream stream) {
  FSVD_TRY(need_init());
  FSVD_TRY(check_ptr(x)); FSVD_TRY(check_ptr(U_up)); FSVD_TRY(check_ptr(V_up));
  FSVD_TRY(check_ptr(U_dn)); FSVD_TRY(check_ptr(V_dn)); FSVD_TRY(check_ptr(y));
  FSVD_TRY(check_opt_ptr(b_up)); FSVD_TRY(check_opt_ptr(b_dn)); FSVD_TRY(check_opt_ptr(resid));
  if (M < 0) return FLASHSVD_ERR_INVALID_ARG;
  FSVD_TRY(check_w8(d)); FSVD_TRY(check_w8(r_up)); FSVD_TRY(check_w8(f)); FSVD_TRY(check_w8(r_dn));
  if (M == 0) return FLASHSVD_OK;
  if (!ffn_stream_covers(d, r_up, f, r_dn)) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  if (M > cur().rows || (long long)M * r_up > (long long)cur().rows * 3 * cur().max_rank)
    return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  return lowrank_ffn(cb(x), cb(U_up), cb(V_up), cb(b_up), cb(U_dn), cb(V_dn), cb(b_dn), cb(resid),
                     (bf16*)y, M, d, r_up, f, r_dn, stream);
}

int flashsvd_dense_kv_decode_attn(const flashsvd_bf16* q,
                                  const flashsvd_bf16* k_new,
                                  const flashsvd_bf16* v_new,
                                  flashsvd_bf16* k_cache,
                                  flashsvd_bf16* v_cache,
                                  const int32_t* cache_seqlens,
                                  flashsvd_bf16* out, int B, int H, int D,
                                  int S_max, float scale,
                                  flashsvd_stream stream) {
  FSVD_TRY(need_init());
  FSVD_TRY(check_ptr(q)); FSVD_TRY(check_ptr(k_cache)); FSVD_TRY(check_ptr(v_cache));
  FSVD_TRY(check_ptr(out));
  if (!cache_seqlens) return FLASHSVD_ERR_INVALID_ARG;
  if ((k_new == nullptr) != (v_new == nullptr)) return FLASHSVD_ERR_INVALID_ARG;
  FSVD_TRY(check_opt_ptr(k_new)); FSVD_TRY(check_opt_ptr(v_new));
  if (B < 0 || H <= 0 || S_max <= 0 || !(scale > 0.f)) return FLASHSVD_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  if (B == 0) return FLASHSVD_OK;
  FSVD_TRY(attn_fits(B, H, D, S_max));
  AttnDecParams a;
  memset(&a, 0, sizeof(a));
  a.q = (const bf16*)q; a.k_new = (const bf16*)k_new; a.v_new = (const bf16*)v_new;
  a.k_cache = (bf16*)k_cache; a.v_cache = (bf16*)v_cache; a.seqlens = cache_seqlens;
  a.out = (bf16*)out; a.B = B; a.H = H; a.D = D; a.S_max = S_max;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.part = cur().apart; a.counters = cur().acounters;
  return attn_decode_launch(a, target_ctas(), stream);
}

int flashsvd_prefill_attn(const flashsvd_bf16* q, const flashsvd_bf16* k_cache,
                          const flashsvd_bf16* v_cache, flashsvd_bf16* out,
                          int B, int S, int H, int D, int S_max, int causal,
                          float scale, flashsvd_stream stream) {
  FSVD_TRY(need_init());
  FSVD_TRY(check_ptr(q)); FSVD_TRY(check_ptr(k_cache)); FSVD_TRY(check_ptr(v_cache));
  FSVD_TRY(check_ptr(out));
  if (B < 0 || S < 0 || H <= 0 || S_max < S || !(scale > 0.f)) return FLASHSVD_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || S == 0) return FLASHSVD_OK;
  AttnPfParams a;
  memset(&a, 0, sizeof(a));
  a.q = (const bf16*)q; a.k = (const bf16*)k_cache; a.v = (const bf16*)v_cache; a.out = (bf16*)out;
  a.B = B; a.S = S; a.H = H; a.D = D; a.S_max = S_max; a.causal = causal ? 1 : 0;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.status = cur().status;
  return attn_prefill_launch(a, stream);
}

int flashsvd_prefill_attn_factorized(const flashsvd_bf16* z_q, const flashsvd_bf16* V_q,
                                     const float* rope_cos, const float* rope_sin,
                                     const flashsvd_bf16* k_cache, const flashsvd_bf16* v_cache,
                                     flashsvd_bf16* out, int B, int S, int H, int D, int S_max, int r,
                                     int causal, float scale, flashsvd_stream stream) {
  FSVD_TRY(need_init());
  FSVD_TRY(check_ptr(z_q)); FSVD_TRY(check_ptr(V_q)); FSVD_TRY(check_ptr(k_cache));
  FSVD_TRY(check_ptr(v_cache)); FSVD_TRY(check_ptr(out));
  FSVD_TRY(check_ptr(rope_cos)); FSVD_TRY(check_ptr(rope_sin));
  if (B < 0 || S < 0 || H <= 0 || r <= 0 || S_max < S || !(scale > 0.f)) return FLASHSVD_ERR_INVALID_ARG;
  if ((D != 64 && D != 128) || r % 64) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || S == 0) return FLASHSVD_OK;
  AttnPfParams a;
  memset(&a, 0, sizeof(a));
  a.k = (const bf16*)k_cache; a.v = (const bf16*)v_cache; a.out = (bf16*)out;
  a.B = B; a.S = S; a.H = H; a.D = D; a.S_max = S_max; a.causal = causal ? 1 : 0;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.status = cur().status;
  a.zq = (const bf16*)z_q; a.ldz = r; a.r = r; a.Vq = (const bf16*)V_q;
  a.rope_cos = rope_cos; a.rope_sin = rope_sin;
  // the caller's z_q is an input: it is not discarded from L2
  return attn_prefill_launch(a, stream);
}

int flashsvd_rmsnorm(const flashsvd_bf16* x, const flashsvd_bf16* g,
                     flashsvd_bf16* y, int M, int d, float eps,
                     flashsvd_stream stream) {
  FSVD_TRY(check_ptr(x)); FSVD_TRY(check_ptr(g)); FSVD_TRY(check_ptr(y));
  if (M < 0 || !(eps >= 0.f)) return FLASHSVD_ERR_INVALID_ARG;
  FSVD_TRY(check_w8(d));
  return rmsnorm_launch((const bf16*)x, (const bf16*)g, (bf16*)y, M, d, eps, stream);
}

int flashsvd_layernorm(const flashsvd_bf16* x, const flashsvd_bf16* g,
                       const flashsvd_bf16* b, flashsvd_bf16* y, int M, int d,
                       float eps, flashsvd_stream stream) {
  FSVD_TRY(check_ptr(x)); FSVD_TRY(check_ptr(g)); FSVD_TRY(check_ptr(b));
  FSVD_TRY(check_ptr(y));
  if (M < 0 || !(eps >= 0.f)) return FLASHSVD_ERR_INVALID_ARG;
  FSVD_TRY(check_w8(d));
  return layernorm_launch((const bf16*)x, (const bf16*)g, (const bf16*)b, (bf16*)y, M, d, eps, stream);
}

int flashsvd_rope_table(float* cos_tab, float* sin_tab, int S_max, int D,
                        float base, flashsvd_stream stream) {
  FSVD_TRY(check_ptr(cos_tab)); FSVD_TRY(check_ptr(sin_tab));
  if (S_max <= 0 || D <= 0 || (D % 2) || !(base > 1.f)) return FLASHSVD_ERR_INVALID_ARG;
  return rope_table_launch(cos_tab, sin_tab, S_max, D, base, stream);
}

int flashsvd_embed(const int32_t* tokens, const flashsvd_bf16* emb,
                   flashsvd_bf16* x, int B, int d, int vocab,
                   flashsvd_stream stream) {
  if (!tokens) return FLASHSVD_ERR_INVALID_ARG;
  FSVD_TRY(check_ptr(emb)); FSVD_TRY(check_ptr(x));
  if (B < 0 || vocab <= 0) return FLASHSVD_ERR_INVALID_ARG;
  FSVD_TRY(check_w8(d));
  return embed_launch(tokens, (const bf16*)emb, (bf16*)x, B, d, vocab, stream);
}

int flashsvd_greedy(const float* logits, int32_t* next_tokens, int M,
                    int vocab, flashsvd_stream stream) {
  if (!logits || !next_tokens || M < 0 || vocab <= 0) return FLASHSVD_ERR_INVALID_ARG;
  return greedy_launch(logits, next_tokens, M, vocab, stream);
}

int flashsvd_advance_seqlens(int32_t* cache_seqlens, int B,
                             flashsvd_stream stream) {
  if (!cache_seqlens || B < 0) return FLASHSVD_ERR_INVALID_ARG;
  if (B == 0) return FLASHSVD_OK;
  return advance_launch(cache_seqlens, B, stream);
}

int flashsvd_layer_forward(const flashsvd_layer* L, flashsvd_bf16* x_inout,
                           flashsvd_bf16* k_cache, flashsvd_bf16* v_cache,
                           const int32_t* cache_seqlens, int B, int S,
                           int S_max, int mode, flashsvd_stream stream) {
  FSVD_TRY(need_init());
  FSVD_TRY(check_layer(L));
  FSVD_TRY(check_ptr(x_inout)); FSVD_TRY(check_ptr(k_cache)); FSVD_TRY(check_ptr(v_cache));
  if (B < 0 || S < 0 || S_max < 1) return FLASHSVD_ERR_INVALID_ARG;
  if (B == 0 || S == 0) return FLASHSVD_OK;
  bf16* x = (bf16*)x_inout;
  bf16* kc = (bf16*)k_cache;
  bf16* vc = (bf16*)v_cache;
  if (mode == FLASHSVD_DECODE) {
    if (L->kind != FLASHSVD_DECODER || S != 1 || !cache_seqlens) return FLASHSVD_ERR_INVALID_ARG;
    if (B > DECODE_MAX_ROWS) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
    if (3 * L->q.r > 3 * cur().max_rank) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
    return layer_decode(L, x, kc, vc, cache_seqlens, B, S_max, stream);
  }
  if (S > S_max) return FLASHSVD_ERR_INVALID_ARG;
  {
    const bool streamed = L->kind == FLASHSVD_ENCODER && ffn_stream_covers(L->d, L->up.r, L->f, L->down.r);
    FSVD_TRY(ensure_scratch(B * S, L->d, streamed ? 0 : L->f));
  }
  if (mode == FLASHSVD_PREFILL_CAUSAL) {
    if (L->kind != FLASHSVD_DECODER) return FLASHSVD_ERR_INVALID_ARG;
    return layer_prefill(L, x, kc, vc, B, S, S_max, stream);
  }
  if (mode == FLASHSVD_ENCODER_BIDIR) {
    if (L->kind != FLASHSVD_ENCODER) return FLASHSVD_ERR_INVALID_ARG;
    return layer_encoder(L, x, kc, vc, B, S, S_max, stream);
  }
  return FLASHSVD_ERR_INVALID_ARG;
}

int flashsvd_capture_begin(flashsvd_stream stream) {
  if (!stream) return FLASHSVD_ERR_INVALID_ARG;  // the legacy stream cannot be captured
  return cuda_status(cudaStreamBeginCapture(stream, cudaStreamCaptureModeThreadLocal));
}

int flashsvd_capture_end(flashsvd_stream stream, flashsvd_graph** graph) {
  if (!stream || !graph) return FLASHSVD_ERR_INVALID_ARG;
  cudaGraph_t g = nullptr;
  FSVD_CUDA(cudaStreamEndCapture(stream, &g));
  return finish_graph(g, graph);
}

int flashsvd_decode_graph_capture(const flashsvd_layer* L,
                                  flashsvd_bf16* x_inout,
                                  flashsvd_bf16* k_cache,
                                  flashsvd_bf16* v_cache,
                                  const int32_t* cache_seqlens, int B,
                                  int S_max, flashsvd_stream stream,
                                  flashsvd_graph** graph) {
  FSVD_TRY(need_init());
  if (!graph || !stream) return FLASHSVD_ERR_INVALID_ARG;
  if (capturing(stream)) return FLASHSVD_ERR_CAPTURE_UNSAFE;
  const int64_t before = g_launches.load();
  FSVD_CUDA(cudaStreamBeginCapture(stream, cudaStreamCaptureModeThreadLocal));
  const int st = flashsvd_layer_forward(L, x_inout, k_cache, v_cache, cache_seqlens, B, 1,
                                        S_max, FLASHSVD_DECODE, stream);
  cudaGraph_t g = nullptr;
  const cudaError_t e = cudaStreamEndCapture(stream, &g);
  g_launches.store(before);
  if (st != FLASHSVD_OK) {
    if (g) cudaGraphDestroy(g);
    return st;
  }
  FSVD_CUDA(e);
  return finish_graph(g, graph);
}

int flashsvd_graph_compose(flashsvd_graph* const* parts, int n_parts,
                           flashsvd_graph** graph) {
  if (!parts || n_parts <= 0 || !graph) return FLASHSVD_ERR_INVALID_ARG;
  cudaGraph_t g = nullptr;
  FSVD_CUDA(cudaGraphCreate(&g, 0));
  cudaGraphNode_t prev = nullptr;
  for (int i = 0; i < n_parts; ++i) {
    if (!parts[i]) { cudaGraphDestroy(g); return FLASHSVD_ERR_INVALID_ARG; }
    cudaGraphNode_t node;
    const cudaError_t e = cudaGraphAddChildGraphNode(&node, g, prev ? &prev : nullptr, prev ? 1 : 0,
                                                     parts[i]->graph);
    if (e != cudaSuccess) { cudaGraphDestroy(g); return cuda_status(e); }
    prev = node;
  }
  return finish_graph(g, graph);
}

int flashsvd_graph_replay(flashsvd_graph* graph, flashsvd_stream stream) {
  if (!graph || !graph->exec) return FLASHSVD_ERR_INVALID_ARG;
  FSVD_CUDA(cudaGraphLaunch(graph->exec, stream));
  g_launches.fetch_add(graph->kernels);
  return FLASHSVD_OK;
}

int flashsvd_graph_kernel_count(const flashsvd_graph* graph) {
  return graph ? graph->kernels : -1;
}

int flashsvd_graph_destroy(flashsvd_graph* graph) {
  if (!graph) return FLASHSVD_ERR_INVALID_ARG;
  if (graph->exec) cudaGraphExecDestroy(graph->exec);
  if (graph->graph) cudaGraphDestroy(graph->graph);
  delete graph;
  return FLASHSVD_OK;
}

}  // extern "C"
