// flashsvd_lowrank_linear_noalloc: the decode-regime factorized linear for
// callers that cannot allocate device memory.
//
// flashsvd_init() obtains its workspace with cudaMalloc.  Some callers cannot
// do that: a plugin running inside a host framework whose allocator owns all
// device memory, or a serving process that must not allocate after start-up.
// This entry point runs the same two split-K GEMV kernels as
// flashsvd_lowrank_linear (M <= 32 path) but takes its scratch -- the fp32
// rank activation z, the split partial sums and the tile counters -- from a
// fixed array in this file, statically placed in device memory when the
// library is loaded.  It allocates nothing and does not need flashsvd_init().
#include <cstring>
#include <mutex>

#include "kernels.h"

namespace fsvd {
namespace {

constexpr int kNaMaxRows = 8;          // M limit
constexpr int kNaMaxRank = 4096;       // r limit
constexpr int kNaMaxWidth = 16384;     // d and n limit
constexpr int kNaPartFloats = 1 << 19; // split partials: 2 MiB
constexpr int kNaCounters = 4096;      // column tiles per launch
constexpr int kNaMaxDevices = 64;

struct NoAllocScratch {
  float z[kNaMaxRows * kNaMaxRank];    // 128 KiB
  float part[kNaPartFloats];
  int counters[kNaCounters];
};

// About 2.2 MiB on every GPU that loads the library, held until exit.  In
// host code this name is a host-side stand-in, never a device address; the
// device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) NoAllocScratch g_noalloc_scratch;

NoAllocScratch* g_scratch_ptr[kNaMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch on the current device (looked up once per
// device, with that device current).
int scratch_for_current_device(NoAllocScratch** out) {
  int dev = 0;
  FSVD_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNaMaxDevices) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    FSVD_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    g_scratch_ptr[dev] = static_cast<NoAllocScratch*>(p);
  }
  *out = g_scratch_ptr[dev];
  return FLASHSVD_OK;
}

// Split-K partial floats one launch of the GEMV needs (same split rule as
// gemv_launch), for rows <= 8.
long long partials_needed(int K, int tiles, int rows, int target) {
  int splits = target / (tiles > 0 ? tiles : 1);
  splits = splits < 1 ? 1 : splits;
  const int max_splits = ceil_div(K, 32);
  splits = splits > max_splits ? max_splits : splits;
  int KC = round_up(ceil_div(K, splits), 32);
  KC = KC > 512 ? 512 : KC;
  splits = ceil_div(K, KC);
  const int mt = rows <= 1 ? 1 : rows <= 2 ? 2 : rows <= 4 ? 4 : 8;
  return (long long)tiles * splits * (mt * 64 + 8);  // split partial stride of the GEMV
}

}  // namespace
}  // namespace fsvd

using namespace fsvd;

extern "C" int flashsvd_lowrank_linear_noalloc(const flashsvd_bf16* x, const flashsvd_bf16* U,
                                               const flashsvd_bf16* V, const flashsvd_bf16* bias,
                                               flashsvd_bf16* y, int M, int d, int r, int n,
                                               flashsvd_stream stream) {
  if (!x || !U || !V || !y) return FLASHSVD_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(U) || !aligned16(V) || !aligned16(y) ||
      (bias && !aligned16(bias)))
    return FLASHSVD_ERR_MISALIGNED;
  if (M < 0 || d <= 0 || r <= 0 || n <= 0) return FLASHSVD_ERR_INVALID_ARG;
  if (d % 8 || r % 8 || n % 8) return FLASHSVD_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return FLASHSVD_OK;
  if (M > kNaMaxRows || r > kNaMaxRank || d > kNaMaxWidth || n > kNaMaxWidth)
    return FLASHSVD_ERR_UNSUPPORTED_SHAPE;

  int dev = 0, sms = 148;
  FSVD_CUDA(cudaGetDevice(&dev));
  FSVD_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const int target = sms * 3;
  const int tiles1 = gemv_tiles_for(MAP_PLAIN, r, 64);
  const int tiles2 = gemv_tiles_for(MAP_PLAIN, n, 64);
  if (tiles1 > kNaCounters || tiles2 > kNaCounters ||
      partials_needed(d, tiles1, M, target) > kNaPartFloats ||
      partials_needed(r, tiles2, M, target) > kNaPartFloats)
    return FLASHSVD_ERR_UNSUPPORTED_SHAPE;

  NoAllocScratch* s = nullptr;
  FSVD_TRY(scratch_for_current_device(&s));
  // The tile counters must start at zero; the kernels return them to zero,
  // but a call that failed part-way may not have.
  FSVD_CUDA(cudaMemsetAsync(s->counters, 0, sizeof(s->counters), stream));

  GvParams p1;
  memset(&p1, 0, sizeof(p1));
  p1.K = d; p1.nprob = 1;
  p1.prob[0].W = reinterpret_cast<const bf16*>(U); p1.prob[0].ldw = r; p1.prob[0].N = r;
  p1.x = reinterpret_cast<const bf16*>(x); p1.ldx = d;
  p1.out32 = s->z; p1.ldo32 = r;
  p1.part = s->part; p1.counters = s->counters;
  p1.part_cap = kNaPartFloats; p1.counters_cap = kNaCounters;
  FSVD_TRY(gemv_launch(p1, PRO_BF16, EPI_F32, MAP_PLAIN, M, target, stream));

  GvParams p2;
  memset(&p2, 0, sizeof(p2));
  p2.K = r; p2.nprob = 1;
  p2.prob[0].W = reinterpret_cast<const bf16*>(V); p2.prob[0].ldw = n; p2.prob[0].N = n;
  p2.a32 = s->z; p2.lda = r;
  p2.out16 = reinterpret_cast<bf16*>(y); p2.ldo16 = n;
  p2.bias = reinterpret_cast<const bf16*>(bias);
  p2.part = s->part; p2.counters = s->counters;
  p2.part_cap = kNaPartFloats; p2.counters_cap = kNaCounters;
  return gemv_launch(p2, PRO_F32, EPI_BF16, MAP_PLAIN, M, target, stream);
}
