// fa_api.cu - the C ABI of libfa.so (declared in include/fa.h): argument validation,
// TMA tensor-map encoding and kernel launches.  No exception crosses this boundary and no
// device memory is allocated here.
#include "fa.h"
#include "fa_debug.cuh"
#include "fa_internal.cuh"
#include "sm100_ptx.cuh"

#include <cudaTypedefs.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <functional>
#include <mutex>
#include <unordered_map>
#include <vector>
#include <algorithm>

namespace fa {

__device__ uint32_t g_fa_status = 0;

#ifdef FA_DEBUG
// Visit counters of the debug build: three blocks of kDebugVisitInts ints (see debug_visits).
__device__ int g_fa_visits[3 * kDebugVisitInts];
#endif

int* debug_visits(int kind) {
#ifdef FA_DEBUG
  static int* cached[64];
  int dev = 0;
  if (kind < 0 || kind > 2 || cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev] + kind * kDebugVisitInts;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_fa_visits) != cudaSuccess) return nullptr;
  if (dev >= 0 && dev < 64) cached[dev] = static_cast<int*>(p);
  return static_cast<int*>(p) + kind * kDebugVisitInts;
#else
  (void)kind;
  return nullptr;
#endif
}

uint32_t* device_status_word() {
  static uint32_t* cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev];
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_fa_status) != cudaSuccess) return nullptr;
  if (dev >= 0 && dev < 64) cached[dev] = static_cast<uint32_t*>(p);
  return static_cast<uint32_t*>(p);
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Per-device check that the current device is an sm_100 part (cached for up to 64 devices).
fa_status_t check_device() {
  static int cached[64];  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev >= 0 && dev < 64 && cached[dev]) return cached[dev] == 1 ? FA_OK : FA_ERR_UNSUPPORTED;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  const bool ok = (major == 10 && minor == 0);
  if (dev >= 0 && dev < 64) cached[dev] = ok ? 1 : 2;
  return ok ? FA_OK : FA_ERR_UNSUPPORTED;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shared shape/scalar validation.  Returns FA_OK and sets *empty when there is nothing to do.
fa_status_t check_shape(int B, int H, int N, int d, float scale, int causal, bool* empty) {
  *empty = false;
  if (B < 0 || H < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const long long bh = (long long)B * H;
  if (bh > INT_MAX) return FA_ERR_INVALID_ARG;
  if (bh == 0 || N == 0) {
    *empty = true;
    return FA_OK;
  }
  // element count must stay far from overflow in every index computation
  if ((long double)bh * N * d >= (long double)(1ull << 62)) return FA_ERR_INVALID_ARG;
  // one CTA per (head, 256 query rows) in the forward, per (head, 128 keys) in the backward
  if (bh * ((N + 127) / 128) > INT_MAX) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// Per-query-tile statistics of the backward: [BH][ceil(N/64)][128] fp32, rounded to 256 bytes.
// Work order of the attention grids.  Under the causal mask a head's query blocks (forward) or
// key tiles (backward) differ in length, so launching the heaviest first shortens the tail; but
// the blocks in flight then spread over every head so ordered, whose streamed operand pair (K, V
// in the forward; Q, dO in the backward) must stay in L2 together.  Heads therefore go in groups:
// inside a group every head's heaviest block goes first, and the group is as many heads as have
// their pairs within kWorkGroupBytes (L2 is 126 MB).  Measured on B200 (step time of forward +
// backward): at B=1 H=32 N=16384 d=128, groups of 4 heads (32 MB) are 2.6 % faster than one head
// (forward 4.8 %, backward key-tile kernel 1.7 %), groups of 8 and 16 lose part or all of it to
// L2 misses; at B=2 H=16 N=4096, groups of 16 beat 4 and all 32 heads by 3.5 % and 1.3 %.
constexpr double kWorkGroupBytes = 32.0 * 1024 * 1024;
int work_group(long long BH, int N, int d, int elem_bytes, int causal) {
  if (!causal) return 1;  // blocks of equal length: a head's blocks together
  const double head_pair = 2.0 * (double)N * d * elem_bytes;
  const long long g = (long long)(kWorkGroupBytes / head_pair);
  return (int)std::max(1LL, std::min(BH, g));
}

size_t ld_bytes(long long bh, int N) {
  const long long tiles = bh * ((N + 63) / 64);
  return ((size_t)tiles * 128 * 4 + 255) & ~(size_t)255;
}

// The backward workspace: the per-tile statistics (ld_bytes), the fp32 dQ accumulator, then a
// 256-byte block whose first two ints are the key-tile kernel's work counter.
constexpr size_t kWorkBytes = 256;
int* work_counter(void* workspace, long long bh, int N, int d) {
  return reinterpret_cast<int*>(reinterpret_cast<char*>(workspace) + ld_bytes(bh, N) + (size_t)bh * N * d * 4);
}

}  // namespace

// Tensor maps depend only on (address, shape, box, element type, swizzle), so encoded maps are
// cached under that key: a map found here is exactly what encoding again would produce.
namespace {
struct TmapKey {
  uintptr_t ptr;
  int BH, N, d, box_inner, box_rows, kind;
  bool operator==(const TmapKey& o) const {
    return ptr == o.ptr && BH == o.BH && N == o.N && d == o.d && box_inner == o.box_inner &&
           box_rows == o.box_rows && kind == o.kind;
  }
};
struct TmapKeyHash {
  size_t operator()(const TmapKey& k) const {
    size_t h = std::hash<uintptr_t>()(k.ptr);
    for (int v : {k.BH, k.N, k.d, k.box_inner, k.box_rows, k.kind}) h = h * 1000003u ^ std::hash<int>()(v);
    return h;
  }
};
std::mutex g_tmap_mu;
std::unordered_map<TmapKey, CUtensorMap, TmapKeyHash> g_tmap_cache;

template <class F>
bool cached_tmap(CUtensorMap* m, const TmapKey& key, F&& encode) {
  {
    std::lock_guard<std::mutex> lock(g_tmap_mu);
    auto it = g_tmap_cache.find(key);
    if (it != g_tmap_cache.end()) {
      *m = it->second;
      return true;
    }
  }
  if (!encode(m)) return false;
  std::lock_guard<std::mutex> lock(g_tmap_mu);
  if (g_tmap_cache.size() >= 4096) g_tmap_cache.clear();
  g_tmap_cache.emplace(key, *m);
  return true;
}
}  // namespace

bool make_tmap_bf16(CUtensorMap* m, const void* ptr, int BH, int N, int d, int box_rows) {
  return cached_tmap(m, TmapKey{reinterpret_cast<uintptr_t>(ptr), BH, N, d, 64, box_rows, 0},
                     [&](CUtensorMap* out) { return encode_tmap_bf16(out, ptr, BH, N, d, box_rows); });
}

bool make_tmap_e4m3(CUtensorMap* m, const void* ptr, int BH, int N, int d, int box_rows) {
  return cached_tmap(m, TmapKey{reinterpret_cast<uintptr_t>(ptr), BH, N, d, 128, box_rows, 3}, [&](CUtensorMap* out) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)d, (cuuint64_t)N * d};
    cuuint32_t box[3] = {128, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(out, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  });
}

bool encode_tmap_bf16(CUtensorMap* m, const void* ptr, int BH, int N, int d, int box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// One thread waits on a phase that never completes; the bounded wait records the timeout.
__global__ void fa_wait_probe_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = ptx::smem_u32(&bar);
  ptx::mbar_init(b, 1);
  ptx::fence_mbar_init();
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try_wait(b, 0)) {
    if (ptx::globaltimer() - t0 > limit_ns) {
      atomicOr(status, FA_DEV_TIMEOUT);
      return;
    }
  }
}

cudaError_t launch_wait_probe(uint32_t* status, uint64_t limit_ns, cudaStream_t stream) {
  fa_wait_probe_kernel<<<1, 1, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

bool make_tmap_f32(CUtensorMap* m, const void* ptr, int BH, int N, int d, int box_inner, int box_rows,
                   bool swizzle128) {
  return cached_tmap(m,
                     TmapKey{reinterpret_cast<uintptr_t>(ptr), BH, N, d, box_inner, box_rows, swizzle128 ? 2 : 1},
                     [&](CUtensorMap* out) {
                       return encode_tmap_f32(out, ptr, BH, N, d, box_inner, box_rows, swizzle128);
                     });
}

bool encode_tmap_f32(CUtensorMap* m, const void* ptr, int BH, int N, int d, int box_inner, int box_rows,
                     bool swizzle128) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)N * d * 4};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_status_string(fa_status_t s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_DEVICE_CHECK: return "FA_ERR_DEVICE_CHECK";
  }
  return "FA_ERR_UNKNOWN";
}

int fa_version(void) { return 100; }

fa_status_t fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                   int N, int d, float scale, int causal, void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, scale, causal, &empty);
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  const int BH = B * H;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_bf16(&tq, q, BH, N, d, 128) || !make_tmap_bf16(&tk, k, BH, N, d, 128) ||
      !make_tmap_bf16(&tv, v, BH, N, d, 128) || !make_tmap_bf16(&to, o, BH, N, d, 32))
    return FA_ERR_CUDA;
  FwdArgs a;
  if (!(a.status = device_status_word())) return FA_ERR_CUDA;
  a.lse = lse;
  a.N = N;
  a.BH = BH;
  a.nqb = (N + 255) / 256;
  a.causal = causal;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  a.nsplit = 1;
  a.group = work_group(BH, N, d, 2, causal);
  if ((long long)a.BH * a.nqb > INT_MAX) return FA_ERR_INVALID_ARG;
  return launch_fwd(d, tq, tk, tv, to, a, (cudaStream_t)stream) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status_t fa_fwd_fp8(const void* q, const void* k, const void* v, const float* descale_q,
                       const float* descale_k, const float* descale_v, void* o, float* lse, int B, int H,
                       int N, int d, float scale, int causal, void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, scale, causal, &empty);
  if (st != FA_OK || empty) return st;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(descale_q, 4) || !aligned(descale_k, 4) || !aligned(descale_v, 4))
    return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  const int BH = B * H;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_e4m3(&tq, q, BH, N, d, 128) || !make_tmap_e4m3(&tk, k, BH, N, d, 128) ||
      !make_tmap_e4m3(&tv, v, BH, N, d, 128) || !make_tmap_bf16(&to, o, BH, N, d, 32))
    return FA_ERR_CUDA;
  FwdArgs a;
  if (!(a.status = device_status_word())) return FA_ERR_CUDA;
  a.lse = lse;
  a.N = N;
  a.BH = BH;
  a.nqb = (N + 255) / 256;
  a.causal = causal;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  a.nsplit = 1;
  a.group = work_group(BH, N, d, 1, causal);
  a.descale_q = descale_q;
  a.descale_k = descale_k;
  a.descale_v = descale_v;
  if ((long long)a.BH * a.nqb > INT_MAX) return FA_ERR_INVALID_ARG;
  return launch_fwd_fp8(d, tq, tk, tv, to, a, (cudaStream_t)stream) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Makespan, in 128-key-block units, of the forward grid with `sp` splits: the CTAs in launch
// order (per head, heavy query blocks first; the splits of an item adjacent) go to whichever
// SM frees up first.  Each CTA costs its key blocks plus a fixed 4 for its prologue and
// epilogue.
static double splitkv_makespan(long long BH, int N, bool causal, int sp, int nsm) {
  const int Tk = (N + 127) / 128, nqb = (N + 255) / 256;
  std::vector<double> sm(nsm, 0.0);  // min-heap of SM finish times
  std::make_heap(sm.begin(), sm.end(), std::greater<double>());
  for (long long bh = 0; bh < BH; ++bh)
    for (int qb = nqb - 1; qb >= 0; --qb) {
      const int n0 = causal ? std::min(Tk, 2 * qb + 1) : Tk;
      const int n1 = (qb * 256 + 128 < N) ? (causal ? std::min(Tk, 2 * qb + 2) : Tk) : 0;
      const int nm = std::max(n0, n1);
      for (int s = 0; s < sp; ++s) {
        const int kb0 = (int)((long long)s * nm / sp), kb1 = (int)((long long)(s + 1) * nm / sp);
        const int w = std::max(std::max(0, std::min(kb1, n0) - kb0), std::max(0, std::min(kb1, n1) - kb0));
        std::pop_heap(sm.begin(), sm.end(), std::greater<double>());
        sm.back() += w + 4.0;
        std::push_heap(sm.begin(), sm.end(), std::greater<double>());
      }
    }
  return *std::max_element(sm.begin(), sm.end());
}

// Split count used when the caller passes num_splits <= 0.  Splitting helps when the grid's
// makespan is set by its longest CTAs rather than by the total work (few heads and causal
// rows of very different lengths); it costs the fp32 partial outputs and the merge, which
// measured 10-20 % of the predicted gain.  So: simulate 1-4 splits and split only if the
// predicted gain is at least 1.25, taking the smallest count within 5 % of the best.
int fa_fwd_splitkv_default_splits(int B, int H, int N, int d, int causal) {
  (void)d;
  if (B <= 0 || H <= 0 || N <= 0) return 1;
  int nsm = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) nsm = v;
  }
  const long long BH = (long long)B * H;
  const long long items = BH * ((N + 255) / 256);
  if (items > 4LL * nsm) return 1;  // several waves: the total work sets the pace
  const int Tk = (N + 127) / 128;
  const double t1 = splitkv_makespan(BH, N, causal != 0, 1, nsm);
  double best = t1;
  double t[5] = {0, t1, 0, 0, 0};
  for (int sp = 2; sp <= 4 && sp <= Tk; ++sp) {
    t[sp] = splitkv_makespan(BH, N, causal != 0, sp, nsm);
    best = std::min(best, t[sp]);
  }
  if (t1 < 1.25 * best) return 1;
  for (int sp = 2; sp <= 4 && sp <= Tk; ++sp)
    if (t[sp] <= 1.05 * best) return sp;
  return 1;
}

static size_t splitkv_o_bytes(long long rows, int d, int sp) {
  return (((size_t)sp * rows * d * 4) + 255) & ~(size_t)255;
}

size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int N, int d, int num_splits) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || num_splits <= 1) return 0;
  const long long rows = (long long)B * H * N;
  return splitkv_o_bytes(rows, d, num_splits) + (size_t)num_splits * rows * 4;
}

fa_status_t fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                           int N, int d, float scale, int causal, int num_splits, void* workspace,
                           size_t workspace_bytes, void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, scale, causal, &empty);
  if (st != FA_OK || empty) return st;
  int sp = num_splits > 0 ? num_splits : fa_fwd_splitkv_default_splits(B, H, N, d, causal);
  const int kblocks = (N + 127) / 128;
  if (sp > kblocks) sp = kblocks;
  if (sp <= 1) return fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, stream);
  if (!q || !k || !v || !o || !lse || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(workspace, 256))
    return FA_ERR_INVALID_ARG;
  if (workspace_bytes < fa_fwd_splitkv_workspace_bytes(B, H, N, d, sp)) return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  const int BH = B * H;
  const long long rows = (long long)BH * N;
  if ((long long)BH * sp > INT_MAX || (long long)BH * ((N + 255) / 256) * sp > INT_MAX) return FA_ERR_INVALID_ARG;
  float* o_part = reinterpret_cast<float*>(workspace);
  float* lse_part = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + splitkv_o_bytes(rows, d, sp));
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_bf16(&tq, q, BH, N, d, 128) || !make_tmap_bf16(&tk, k, BH, N, d, 128) ||
      !make_tmap_bf16(&tv, v, BH, N, d, 128) || !make_tmap_f32(&to, o_part, BH * sp, N, d, 32, 32, true))
    return FA_ERR_CUDA;
  FwdArgs a;
  if (!(a.status = device_status_word())) return FA_ERR_CUDA;
  a.lse = lse_part;
  a.N = N;
  a.BH = BH;
  a.nqb = (N + 255) / 256;
  a.causal = causal;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  a.nsplit = sp;
  a.group = work_group(BH, N, d, 2, causal);
  cudaStream_t s = (cudaStream_t)stream;
  if (launch_fwd(d, tq, tk, tv, to, a, s) != cudaSuccess) return FA_ERR_CUDA;
  if (launch_fwd_merge(o_part, lse_part, o, lse, sp, rows, d, s) != cudaSuccess) return FA_ERR_CUDA;
  return FA_OK;
}

fa_status_t fa_fwd_partial(const void* q, const void* k, const void* v, float* o_part, float* lse_part,
                           int B, int H, int N, int d, float scale, int causal, void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, scale, causal, &empty);
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !o_part || !lse_part) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o_part, 16) || !aligned(lse_part, 4))
    return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  const int BH = B * H;
  if ((long long)BH * ((N + 255) / 256) > INT_MAX) return FA_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_bf16(&tq, q, BH, N, d, 128) || !make_tmap_bf16(&tk, k, BH, N, d, 128) ||
      !make_tmap_bf16(&tv, v, BH, N, d, 128) || !make_tmap_f32(&to, o_part, BH, N, d, 32, 32, true))
    return FA_ERR_CUDA;
  FwdArgs a;
  if (!(a.status = device_status_word())) return FA_ERR_CUDA;
  a.lse = lse_part;
  a.N = N;
  a.BH = BH;
  a.nqb = (N + 255) / 256;
  a.causal = causal;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  a.nsplit = 1;
  a.group = work_group(BH, N, d, 2, causal);
  return launch_fwd_partial(d, tq, tk, tv, to, a, (cudaStream_t)stream) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status_t fa_fwd_carry(const void* q, const void* k, const void* v, float* o_part, float* lse_part, void* o,
                         float* lse, int B, int H, int N, int d, float scale, int causal, int flags,
                         void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, scale, causal, &empty);
  if (st != FA_OK || empty) return st;
  if (flags & ~(FA_CARRY_IN | FA_CARRY_FINAL)) return FA_ERR_INVALID_ARG;
  const bool in = (flags & FA_CARRY_IN) != 0, fin = (flags & FA_CARRY_FINAL) != 0;
  if (!q || !k || !v || !o_part || !lse_part || (fin && (!o || !lse))) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o_part, 16) || !aligned(lse_part, 4) ||
      (fin && (!aligned(o, 16) || !aligned(lse, 4))))
    return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  const int BH = B * H;
  if ((long long)BH * ((N + 255) / 256) > INT_MAX) return FA_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_bf16(&tq, q, BH, N, d, 128) || !make_tmap_bf16(&tk, k, BH, N, d, 128) ||
      !make_tmap_bf16(&tv, v, BH, N, d, 128) ||
      !(fin ? make_tmap_bf16(&to, o, BH, N, d, 32) : make_tmap_f32(&to, o_part, BH, N, d, 32, 32, true)))
    return FA_ERR_CUDA;
  FwdArgs a;
  if (!(a.status = device_status_word())) return FA_ERR_CUDA;
  a.lse = fin ? lse : lse_part;
  a.N = N;
  a.BH = BH;
  a.nqb = (N + 255) / 256;
  a.causal = causal;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  a.nsplit = 1;
  a.group = work_group(BH, N, d, 2, causal);
  if (in) {  // each CTA reads its rows' carried result before it writes them
    a.carry_o = o_part;
    a.carry_lse = lse_part;
  }
  const cudaError_t e = fin ? launch_fwd(d, tq, tk, tv, to, a, (cudaStream_t)stream)
                            : launch_fwd_partial(d, tq, tk, tv, to, a, (cudaStream_t)stream);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status_t fa_merge_partials(const float* o_parts, const float* lse_parts, int nparts, void* o, float* lse,
                              int B, int H, int N, int d, void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, 1.0f, 0, &empty);
  if (st != FA_OK || empty) return st;
  if (nparts < 1 || nparts > 1024) return FA_ERR_INVALID_ARG;
  if (!o_parts || !lse_parts || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned(o_parts, 16) || !aligned(lse_parts, 4) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  const long long rows = (long long)B * H * N;
  return launch_fwd_merge(o_parts, lse_parts, o, lse, nparts, rows, d, (cudaStream_t)stream) == cudaSuccess
             ? FA_OK
             : FA_ERR_CUDA;
}

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return 0;
  const long long rows = (long long)B * H * N;
  return ld_bytes((long long)B * H, N) + (size_t)rows * d * 4 + kWorkBytes;
}

// The key-tile kernel of fa_bwd on prepared statistics (d = 64 or 128): bf16 dK, dV stored (or,
// with dk_acc set, scale * dK and dV added into fp32 accumulators), dQ added into the
// workspace's fp32 accumulator.  Arguments are checked by the callers.
static fa_status_t bwd_main_dq(const void* q, const void* k, const void* v, const void* dO, void* workspace,
                               void* dk, void* dv, int BH, int N, int d, float scale, int causal, cudaStream_t s,
                               float* dk_acc = nullptr, float* dv_acc = nullptr, bool acc_overwrite = false) {
  float* ld = reinterpret_cast<float*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + ld_bytes(BH, N));
  CUtensorMap tq, tk, tv, tdo, tdk, tdv, tdq;
  if (!make_tmap_bf16(&tq, q, BH, N, d, 64) || !make_tmap_bf16(&tk, k, BH, N, d, 128) ||
      !make_tmap_bf16(&tv, v, BH, N, d, 128) || !make_tmap_bf16(&tdo, dO, BH, N, d, 64) ||
      !make_tmap_f32(&tdq, dq_acc, BH, N, d, 32, 64 - kBwdDqRedRows))
    return FA_ERR_CUDA;
  if (dk_acc == nullptr) {
    if (!make_tmap_bf16(&tdk, dk, BH, N, d, 32) || !make_tmap_bf16(&tdv, dv, BH, N, d, 32)) return FA_ERR_CUDA;
  } else {
    tdk = tk;  // accumulate mode: the bf16 store maps are not used; any valid map fills them
    tdv = tv;
  }
  BwdArgs a;
  if (!(a.status = device_status_word())) return FA_ERR_CUDA;
  a.lse = nullptr;
  a.ld = ld;
  a.dq_acc = dq_acc;
  a.dk_acc = dk_acc;
  a.dv_acc = dv_acc;
  a.acc_overwrite = acc_overwrite ? 1 : 0;
  a.N = N;
  a.BH = BH;
  a.causal = causal;
  a.scale = scale;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  a.group = work_group(BH, N, d, 2, causal);
  a.work = work_counter(workspace, BH, N, d);
  cudaError_t e = launch_bwd_main(d, tq, tk, tv, tdo, tdk, tdv, tdq, a, s);
  if (e == cudaErrorNotSupported) return FA_ERR_UNSUPPORTED;
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

static fa_status_t check_bwd_io(const void* q, const void* k, const void* v, const void* dO, const void* dk,
                                const void* dv, const void* workspace, size_t workspace_bytes, int B, int H,
                                int N, int d) {
  if (!q || !k || !v || !dO || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(dO, 16) || !aligned(dk, 16) ||
      !aligned(dv, 16) || !aligned(workspace, 256))
    return FA_ERR_INVALID_ARG;
  if (workspace_bytes < fa_bwd_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

fa_status_t fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                   const float* lse, void* dq, void* dk, void* dv, void* workspace,
                   size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
                   void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, scale, causal, &empty);
  if (st != FA_OK || empty) return st;
  if ((st = check_bwd_io(q, k, v, dO, dk, dv, workspace, workspace_bytes, B, H, N, d)) != FA_OK) return st;
  if (!o || !lse || !dq || !aligned(o, 16) || !aligned(dq, 16) || !aligned(lse, 4)) return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  const int BH = B * H;
  const long long rows = (long long)BH * N;
  float* ld = reinterpret_cast<float*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + ld_bytes(BH, N));
  cudaStream_t s = (cudaStream_t)stream;
  if (launch_bwd_pre(o, dO, lse, ld, dq_acc, work_counter(workspace, BH, N, d), BH, N, d, s) != cudaSuccess)
    return FA_ERR_CUDA;
  if ((st = bwd_main_dq(q, k, v, dO, workspace, dk, dv, BH, N, d, scale, causal, s)) != FA_OK) return st;
  if (launch_bwd_post(dq_acc, dq, rows * d, scale, s) != cudaSuccess) return FA_ERR_CUDA;
  return FA_OK;
}

fa_status_t fa_bwd_main(const void* q, const void* k, const void* v, const void* dO, void* workspace,
                        size_t workspace_bytes, void* dk, void* dv, int B, int H, int N, int d, float scale,
                        int causal, void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, scale, causal, &empty);
  if (st != FA_OK || empty) return st;
  if ((st = check_bwd_io(q, k, v, dO, dk, dv, workspace, workspace_bytes, B, H, N, d)) != FA_OK) return st;
  if ((st = check_device()) != FA_OK) return st;
  return bwd_main_dq(q, k, v, dO, workspace, dk, dv, B * H, N, d, scale, causal, (cudaStream_t)stream);
}

fa_status_t fa_bwd_dq_post(const void* workspace, size_t workspace_bytes, void* dq, int B, int H, int N, int d,
                           float scale, void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, scale, 0, &empty);
  if (st != FA_OK || empty) return st;
  if (!workspace || !dq || !aligned(workspace, 256) || !aligned(dq, 16)) return FA_ERR_INVALID_ARG;
  if (workspace_bytes < fa_bwd_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  const long long rows = (long long)B * H * N;
  const float* dq_acc =
      reinterpret_cast<const float*>(reinterpret_cast<const char*>(workspace) + ld_bytes((long long)B * H, N));
  return launch_bwd_post(dq_acc, dq, rows * d, scale, (cudaStream_t)stream) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status_t fa_bwd_prepare(const void* o, const void* dO, const float* lse, void* workspace, size_t workspace_bytes,
                           int B, int H, int N, int d, void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, 1.0f, 0, &empty);
  if (st != FA_OK || empty) return st;
  if (!o || !dO || !lse || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned(o, 16) || !aligned(dO, 16) || !aligned(lse, 4) || !aligned(workspace, 256)) return FA_ERR_INVALID_ARG;
  if (workspace_bytes < fa_bwd_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  const int BH = B * H;
  float* ld = reinterpret_cast<float*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + ld_bytes(BH, N));
  return launch_bwd_pre(o, dO, lse, ld, dq_acc, work_counter(workspace, BH, N, d), BH, N, d,
                        (cudaStream_t)stream) == cudaSuccess ? FA_OK
                                                                                                : FA_ERR_CUDA;
}

fa_status_t fa_bwd_accumulate(const void* q, const void* k, const void* v, const void* dO, void* workspace,
                              size_t workspace_bytes, float* dk_acc, float* dv_acc, int B, int H, int N, int d,
                              float scale, int causal, void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, scale, causal, &empty);
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !dO || !workspace || !dk_acc || !dv_acc) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(dO, 16) || !aligned(workspace, 256) ||
      !aligned(dk_acc, 16) || !aligned(dv_acc, 16))
    return FA_ERR_INVALID_ARG;
  if (workspace_bytes < fa_bwd_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  return bwd_main_dq(q, k, v, dO, workspace, nullptr, nullptr, B * H, N, d, scale, causal, (cudaStream_t)stream,
                       dk_acc, dv_acc);
}

fa_status_t fa_bwd_contribute(const void* q, const void* k, const void* v, const void* dO, void* workspace,
                              size_t workspace_bytes, float* dk_out, float* dv_out, int B, int H, int N, int d,
                              float scale, int causal, void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, scale, causal, &empty);
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !dO || !workspace || !dk_out || !dv_out) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(dO, 16) || !aligned(workspace, 256) ||
      !aligned(dk_out, 16) || !aligned(dv_out, 16))
    return FA_ERR_INVALID_ARG;
  if (workspace_bytes < fa_bwd_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  return bwd_main_dq(q, k, v, dO, workspace, nullptr, nullptr, B * H, N, d, scale, causal, (cudaStream_t)stream,
                     dk_out, dv_out, true);
}

fa_status_t fa_bwd_finish(const void* workspace, size_t workspace_bytes, const float* dk_acc, const float* dv_acc,
                          void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, scale, 0, &empty);
  if (st != FA_OK || empty) return st;
  if (!workspace || !dk_acc || !dv_acc || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (!aligned(workspace, 256) || !aligned(dk_acc, 16) || !aligned(dv_acc, 16) || !aligned(dq, 16) ||
      !aligned(dk, 16) || !aligned(dv, 16))
    return FA_ERR_INVALID_ARG;
  if (workspace_bytes < fa_bwd_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  const long long elems = (long long)B * H * N * d;
  const float* dq_acc =
      reinterpret_cast<const float*>(reinterpret_cast<const char*>(workspace) + ld_bytes((long long)B * H, N));
  cudaStream_t s = (cudaStream_t)stream;
  if (launch_bwd_post(dq_acc, dq, elems, scale, s) != cudaSuccess) return FA_ERR_CUDA;
  if (launch_bwd_post(dk_acc, dk, elems, 1.0f, s) != cudaSuccess) return FA_ERR_CUDA;
  if (launch_bwd_post(dv_acc, dv, elems, 1.0f, s) != cudaSuccess) return FA_ERR_CUDA;
  return FA_OK;
}

fa_status_t fa_bwd_acc_add(float* acc, const float* x, int B, int H, int N, int d, void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, 1.0f, 0, &empty);
  if (st != FA_OK || empty) return st;
  if (!acc || !x || !aligned(acc, 16) || !aligned(x, 16)) return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  const long long elems = (long long)B * H * N * d;
  return launch_acc_add(acc, x, elems, (cudaStream_t)stream) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status_t fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                 const float* lse, void* dq, void* dk, void* dv, void* workspace,
                                 size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
                                 void* stream) {
  bool empty = false;
  fa_status_t st = check_shape(B, H, N, d, scale, causal, &empty);
  if (st != FA_OK || empty) return st;
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dO, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4) || !aligned(workspace, 256))
    return FA_ERR_INVALID_ARG;
  if (workspace_bytes < fa_bwd_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
  if ((st = check_device()) != FA_OK) return st;
  const int BH = B * H;
  float* ld = reinterpret_cast<float*>(workspace);
  cudaStream_t s = (cudaStream_t)stream;
  // main kernel (dK, dV): Q/dO in 64-row boxes, K/V in 128-row boxes
  CUtensorMap tq64, tk128, tv128, tdo64, tdk, tdv;
  // dQ kernel: Q/dO in 128-row boxes, K/V in 64-row boxes, dQ stored in 32-row boxes
  CUtensorMap tq128, tk64, tv64, tdo128, tdq;
  if (!make_tmap_bf16(&tq64, q, BH, N, d, 64) || !make_tmap_bf16(&tk128, k, BH, N, d, 128) ||
      !make_tmap_bf16(&tv128, v, BH, N, d, 128) || !make_tmap_bf16(&tdo64, dO, BH, N, d, 64) ||
      !make_tmap_bf16(&tdk, dk, BH, N, d, 32) || !make_tmap_bf16(&tdv, dv, BH, N, d, 32) ||
      !make_tmap_bf16(&tq128, q, BH, N, d, 128) || !make_tmap_bf16(&tk64, k, BH, N, d, 64) ||
      !make_tmap_bf16(&tv64, v, BH, N, d, 64) || !make_tmap_bf16(&tdo128, dO, BH, N, d, 128) ||
      !make_tmap_bf16(&tdq, dq, BH, N, d, 32))
    return FA_ERR_CUDA;
  BwdArgs a;
  if (!(a.status = device_status_word())) return FA_ERR_CUDA;
  a.lse = lse;
  a.ld = ld;
  a.dq_acc = nullptr;
  a.N = N;
  a.BH = BH;
  a.causal = causal;
  a.scale = scale;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  a.group = work_group(BH, N, d, 2, causal);
  a.work = work_counter(workspace, BH, N, d);
  if (launch_bwd_pre(o, dO, lse, ld, nullptr, a.work, BH, N, d, s) != cudaSuccess) return FA_ERR_CUDA;
  if (launch_bwd_main(d, tq64, tk128, tv128, tdo64, tdk, tdv, tdk, a, s, false) != cudaSuccess) return FA_ERR_CUDA;
  if (launch_bwd_dq(d, tq128, tk64, tv64, tdo128, tdq, a, s) != cudaSuccess) return FA_ERR_CUDA;
  return FA_OK;
}

fa_status_t fa_selftest_wait_timeout(int limit_ms, void* stream) {
  if (limit_ms < 1 || limit_ms > 1000) return FA_ERR_INVALID_ARG;
  uint32_t* status = device_status_word();
  if (!status) return FA_ERR_CUDA;
  return launch_wait_probe(status, (uint64_t)limit_ms * 1000000ull, (cudaStream_t)stream) == cudaSuccess
             ? FA_OK
             : FA_ERR_CUDA;
}

fa_status_t fa_get_device_status(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return FA_ERR_CUDA;
  uint32_t h = 0;
  const uint32_t zero = 0;
  if (cudaMemcpyFromSymbol(&h, g_fa_status, sizeof(h)) != cudaSuccess) return FA_ERR_CUDA;
  if (h != 0 && cudaMemcpyToSymbol(g_fa_status, &zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
  if (h & FA_DEV_TIMEOUT) return FA_ERR_TIMEOUT;
  return h ? FA_ERR_DEVICE_CHECK : FA_OK;
}

int fa_debug_build(void) {
#ifdef FA_DEBUG
  return 1;
#else
  return 0;
#endif
}

fa_status_t fa_debug_visits(int* counts, size_t n, int clear, void* stream) {
#ifdef FA_DEBUG
  if (n > (size_t)(3 * kDebugVisitInts) || (n > 0 && counts == nullptr)) return FA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return FA_ERR_CUDA;
  int* base = debug_visits(0);
  if (base == nullptr) return FA_ERR_CUDA;
  if (n > 0 && cudaMemcpy(counts, base, n * sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_CUDA;
  if (clear && cudaMemset(base, 0, (size_t)(3 * kDebugVisitInts) * sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (clear && cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
  return FA_OK;
#else
  (void)counts, (void)n, (void)clear, (void)stream;
  return FA_ERR_UNSUPPORTED;
#endif
}

}  // extern "C"
