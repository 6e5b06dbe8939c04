// Host side of the batched Muon update: argument checks, launch plans,
// scratch layout, TMA descriptors and the C ABI declared in include/dmuon.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <list>
#include <map>
#include <memory>
#include <mutex>
#include <string>
#include <unordered_set>
#include <utility>
#include <vector>

#include "dmuon.h"
#include "kernels.cuh"

namespace dmuon {

__device__ int g_device_error = 0;

namespace {

// ------------------------------------------------------------------ errors
thread_local std::string t_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(DMUON_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

std::mutex g_mu;
int g_fail_allocs = 0;
int64_t g_launches = 0;   // kernels this library has launched

// Device memory of the library (launch plans, scratch arenas) comes from one
// memory pool per device, allocated and freed in stream order: no call
// blocks on, or synchronises, the device.  The pool keeps freed memory for
// reuse (release threshold: unlimited) until dmuon_release_cache().
cudaError_t lib_malloc_async(void** p, size_t bytes, cudaMemPool_t pool, cudaStream_t st) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_fail_allocs > 0) {
      --g_fail_allocs;
      *p = nullptr;
      return cudaErrorMemoryAllocation;
    }
  }
  return cudaMallocFromPoolAsync(p, bytes, pool, st);
}

// ------------------------------------------------------------------ driver
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 2-D row-major tensor: `inner` elements per row (contiguous), `outer` rows,
// row pitch `pitch_elems`; box `box_inner` x `box_outer`, 128-byte swizzle,
// zero fill out of bounds.
bool encode_2d(CUtensorMap* map, int dtype, void* base, uint64_t inner, uint64_t outer,
               uint64_t pitch_elems, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const int eb = dtype == DMUON_BF16 ? 2 : 4;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_elems * eb};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype == DMUON_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 matrix with `cols` a multiple of 64 seen as 3-D: {64 columns within a
// block, rows, blocks of 64 columns}, box {64, 64, 4}, 128-byte swizzle.  One
// box is the 64 x 256 MN-major operand tile that four 2-D boxes would bring,
// in the same shared-memory layout (four 8 KB blocks); in the last column
// tile, blocks past the last column are out of bounds and arrive as zeros.
bool encode_mn3d(CUtensorMap* map, void* base, uint64_t cols, uint64_t rows, uint64_t pitch_elems,
                 uint32_t blocks = 4) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || cols % 64 != 0) return false;
  cuuint64_t dims[3] = {64, rows, cols / 64};
  cuuint64_t strides[2] = {pitch_elems * 2, 128};
  cuuint32_t box[3] = {64, 64, blocks};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ inputs
struct MatIn {
  void* W;
  const void* G;
  float* buf;
  int64_t rows, cols;
  int pdt, gdt;
  int mode;
  float lr_mult = 1.0f;   // per-matrix factor on lr
  std::vector<const void*> gr;   // with more than one: the ranks' gradient buffers to average
};

// Scalars and switches of one call.
struct StepOpts {
  float lr = 0.0f, mu = 0.0f, wd = 0.0f;
  int nesterov = 0, steps = 0;
  float ca = 1.5f, cb = -0.5f;      // cubic coefficients
  float cc = 0.0f;                  // != 0: quintic X <- ca X + cb A X + cc A A X
  int lr_scale = DMUON_LR_PLAIN;
  float max_norm = 0.0f;            // > 0: global-norm gradient clipping
  float* norm_out = nullptr;        // device pointer for the pre-clip norm
};

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t b) { return cdiv(a, b) * b; }
inline size_t align_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

int elem_bytes(int dt) { return dt == DMUON_BF16 ? 2 : 4; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_matrix(const MatIn& x, int i) {
  if (x.rows < 1 || x.cols < 1)
    return fail(DMUON_ERR_INVALID_ARG, "matrix %d: rows and cols must be >= 1 (got %lld x %lld)", i,
                (long long)x.rows, (long long)x.cols);
  if ((x.pdt != DMUON_BF16 && x.pdt != DMUON_F32) || (x.gdt != DMUON_BF16 && x.gdt != DMUON_F32))
    return fail(DMUON_ERR_UNSUPPORTED, "matrix %d: dtype must be DMUON_BF16 or DMUON_F32", i);
  const int64_t m = std::min(x.rows, x.cols), n = std::max(x.rows, x.cols);
  if (m > DMUON_MAX_M || n > DMUON_MAX_N)
    return fail(DMUON_ERR_UNSUPPORTED, "matrix %d: %lld x %lld exceeds the size limits", i,
                (long long)x.rows, (long long)x.cols);
  if (!x.W || !x.G)
    return fail(DMUON_ERR_INVALID_ARG, "matrix %d: NULL pointer", i);
  if (x.mode == kModeMuon && !x.buf)
    return fail(DMUON_ERR_INVALID_ARG, "matrix %d: NULL momentum buffer", i);
  if (!aligned(x.W, elem_bytes(x.pdt)) || !aligned(x.G, elem_bytes(x.gdt)) ||
      (x.buf && !aligned(x.buf, 4)))
    return fail(DMUON_ERR_INVALID_ARG, "matrix %d: pointer not aligned to its element size", i);
  return DMUON_OK;
}

// ------------------------------------------------------------------ layout
// Scratch per matrix: X0 [, X1] [, A], then per group the tile partials and
// the per-matrix scales.  Every region starts on a 1024-byte boundary.
struct MatLayout {
  int64_t m, n, ldx, lda;
  size_t x0, x1, a;        // byte offsets in the workspace (x1/a = SIZE_MAX if unused)
  size_t p;                // quintic: P = b A + c A A (SIZE_MAX if unused)
  size_t o0, o1;           // tf32 operand copies of X0/X1 (fp32 only; else == x0/x1)
  int64_t ptiles, ptiles_c;
};
struct GroupLayout {
  int dtype;
  std::vector<int> idx;    // indices into the input matrix array
  size_t partials, scales; // byte offsets
  size_t gpartials;        // byte offset of the gradient-norm partials (double per item)
  int64_t ptiles;
};
struct Layout {
  std::vector<MatLayout> mats;   // parallel to the input matrices
  std::vector<GroupLayout> groups;
  size_t clip = 0;               // byte offset of {clip coefficient, gradient norm}
  size_t bytes = 0;
};

Layout make_layout(const std::vector<MatIn>& in, int steps, bool quintic = false) {
  Layout L;
  L.mats.resize(in.size());
  size_t off = 0;
  for (int dt : {DMUON_BF16, DMUON_F32}) {
    GroupLayout g;
    g.dtype = dt;
    g.ptiles = 0;
    for (size_t i = 0; i < in.size(); ++i)
      if (in[i].pdt == dt) g.idx.push_back(static_cast<int>(i));
    if (g.idx.empty()) continue;
    const int eb = elem_bytes(dt);
    const int64_t q = 16 / eb;   // 16-byte row pitch granularity
    for (int i : g.idx) {
      MatLayout& ml = L.mats[i];
      ml.m = std::min(in[i].rows, in[i].cols);
      ml.n = std::max(in[i].rows, in[i].cols);
      ml.ldx = round_up(ml.n, q);
      ml.lda = round_up(ml.m, q);
      const size_t xb = static_cast<size_t>(ml.m) * ml.ldx * eb;
      const size_t ab = static_cast<size_t>(ml.m) * ml.lda * eb;
      ml.x0 = off; off = align_up(off + xb, 1024);
      ml.x1 = SIZE_MAX; ml.a = SIZE_MAX;
      if (steps >= 2) { ml.x1 = off; off = align_up(off + xb, 1024); }
      ml.o0 = ml.x0; ml.o1 = ml.x1;
      if (dt == DMUON_F32 && steps >= 1) {
        ml.o0 = off; off = align_up(off + xb, 1024);
        if (steps >= 2) { ml.o1 = off; off = align_up(off + xb, 1024); }
      }
      if (steps >= 1) { ml.a = off; off = align_up(off + ab, 1024); }
      ml.p = SIZE_MAX;
      if (steps >= 1 && quintic) { ml.p = off; off = align_up(off + ab, 1024); }
      // Prologue work items: flat chunks, or kTR x kTC tiles when transposed.
      if (in[i].rows > in[i].cols) {
        ml.ptiles_c = cdiv(in[i].cols, kTC);
        ml.ptiles = cdiv(in[i].rows, kTR) * ml.ptiles_c;
      } else {
        ml.ptiles_c = 0;
        ml.ptiles = cdiv(in[i].rows * in[i].cols, kFlatChunk);
      }
      g.ptiles += ml.ptiles;
    }
    g.partials = off; off = align_up(off + sizeof(float) * g.ptiles, 1024);
    g.scales = off; off = align_up(off + sizeof(float) * g.idx.size(), 1024);
    g.gpartials = off; off = align_up(off + sizeof(double) * g.ptiles, 1024);
    L.groups.push_back(std::move(g));
  }
  L.clip = off; off = align_up(off + 2 * sizeof(float), 1024);
  L.bytes = off;
  return L;
}

// ------------------------------------------------------------------ plans
struct GroupPlan {
  int dtype;
  bool ranks = false;     // some matrix averages several ranks' gradients
  bool g_bf16 = true;     // every gradient of the group is bf16
  int nmat;
  int first;              // first MatDesc index of the group
  int64_t ptiles;
  int syrk_tiles, gemm_tiles, square_tiles;
  bool syrk256 = true;    // SYRK by syrk256_kernel (256 x 256 tiles), else ns_stage_kernel<kSyrk>
  bool gemm_pair = false; // GEMM by gemm_pair_kernel (256 x 256 tiles on CTA pairs)
  bool square256 = false; // quintic SQUARE by syrk256_kernel<kSquare> (pair groups whose A has a 3-D view)
  const int* syrk_order; const int* syrk_prefix;
  const int* gemm_order; const int* gemm_prefix;
  const int* square_prefix;   // SQUARE tiles along gemm_order (quintic plans)
  const int64_t* pprefix;
  float* partials;
  double* gpartials;
};

// The caller's addresses of one matrix, as a plan's device descriptors hold them.
struct PtrSet {
  void* W = nullptr;
  const void* G = nullptr;
  float* buf = nullptr;
  int vec4 = 0;
  bool operator==(const PtrSet& o) const { return W == o.W && G == o.G && buf == o.buf && vec4 == o.vec4; }
};

// A launch plan depends on the shapes, types, options class and scratch
// address of a call, not on the caller's tensor addresses: those are written
// into the plan's descriptors by a small patch kernel, in stream order, when
// they differ from the ones the descriptors hold.
struct Plan {
  std::vector<uint8_t> key;
  uint64_t hash = 0;
  int device = 0;
  void* dmem = nullptr;           // pool memory (freed in stream order on eviction)
  const MatDesc* d_mats = nullptr;
  const MatMaps* d_maps = nullptr;
  float* clip = nullptr;          // workspace: {clip coefficient, gradient norm}
  bool quintic = false;
  std::vector<GroupPlan> groups;
  std::vector<int> desc_of;       // input matrix -> descriptor index
  std::vector<PtrSet> cur;        // per descriptor: the addresses its device copy holds
  bool captured = false;          // used in a graph capture: replays rewrite the addresses
  cudaEvent_t last = nullptr;     // recorded after the latest work that used the plan
  cudaStream_t last_st = nullptr; // ... on this stream
  ~Plan() {
    if (dmem) cudaFree(dmem);
    if (last) cudaEventDestroy(last);
  }
};

struct DeviceInfo {
  bool ready = false;
  int sms = 0;
  int pair_clusters = 0;   // co-resident two-CTA clusters of gemm_pair_kernel (0: not used)
  int* err = nullptr;
  cudaMemPool_t pool = nullptr;
};
DeviceInfo g_dev[64];
std::list<std::unique_ptr<Plan>> g_plans;   // most recently used first
constexpr size_t kMaxPlans = 64;   // > the groups of one call (<= 32): a call never evicts its own plans

struct Arena {
  void* ptr = nullptr;
  size_t bytes = 0;
};
std::map<std::pair<int, cudaStream_t>, Arena> g_arenas;
// Library memory whose stream-ordered free could not be enqueued (it may
// still be in use): freed by dmuon_release_cache after its device sync.
std::vector<void*> g_parked;

// Frees library memory after the work enqueued on `st` so far (and, with
// `after`, after that event too).  Never frees memory that may be in use:
// when the free cannot be enqueued, the memory is parked instead.
void free_in_order(void* p, cudaStream_t st, cudaEvent_t after = nullptr) {
  cudaError_t e = after ? cudaStreamWaitEvent(st, after, 0) : cudaSuccess;
  if (e == cudaSuccess) e = cudaFreeAsync(p, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    g_parked.push_back(p);
  }
}

// DMUON_LOG set to anything but "0": one stderr line per launch plan built.
bool log_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("DMUON_LOG");
    return v != nullptr && v[0] != '\0' && !(v[0] == '0' && v[1] == '\0');
  }();
  return on;
}

uint64_t fnv1a(const uint8_t* p, size_t n) {
  uint64_t h = 1469598103934665603ull;
  for (size_t i = 0; i < n; ++i) { h ^= p[i]; h *= 1099511628211ull; }
  return h;
}

template <typename T>
void put(std::vector<uint8_t>& v, const T& x) {
  const uint8_t* p = reinterpret_cast<const uint8_t*>(&x);
  v.insert(v.end(), p, p + sizeof(T));
}

int device_setup(int dev) {
  if (dev < 0 || dev >= 64) return fail(DMUON_ERR_CUDA, "device index %d out of range", dev);
  DeviceInfo& d = g_dev[dev];
  if (d.ready) return DMUON_OK;
  cudaError_t e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(DMUON_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                major, minor);
  e = cudaGetSymbolAddress(reinterpret_cast<void**>(&d.err), g_device_error);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
  const void* ks[] = {
      reinterpret_cast<const void*>(&ns_stage_kernel<kSyrk, __nv_bfloat16>),
      reinterpret_cast<const void*>(&ns_stage_kernel<kGemm, __nv_bfloat16>),
      reinterpret_cast<const void*>(&ns_stage_kernel<kSyrk, float>),
      reinterpret_cast<const void*>(&ns_stage_kernel<kGemm, float>),
      reinterpret_cast<const void*>(&ns_stage_kernel<kSquare, __nv_bfloat16>),
      reinterpret_cast<const void*>(&ns_stage_kernel<kSquare, float>)};
  for (const void* k : ks) {
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kNsSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(smem)");
  }
  const void* ks2[] = {reinterpret_cast<const void*>(&syrk256_kernel<__nv_bfloat16>),
                       reinterpret_cast<const void*>(&syrk256_kernel<float>),
                       reinterpret_cast<const void*>(&syrk256_kernel<__nv_bfloat16, kSquare>)};
  for (const void* k : ks2) {
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kS2SmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(smem)");
  }
  {
    const void* k = reinterpret_cast<const void*>(&gemm_pair_kernel);
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kG2SmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(smem)");
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(2 * static_cast<unsigned>(d.sms / 2), 1, 1);
    cfg.blockDim = dim3(kNsThreads, 1, 1);
    cfg.dynamicSmemBytes = kG2SmemBytes;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int nc = 0;
    // Without a usable answer the pair GEMM is not used.
    if (cudaOccupancyMaxActiveClusters(&nc, k, &cfg) != cudaSuccess) {
      cudaGetLastError();
      nc = 0;
    }
    d.pair_clusters = std::min(nc, d.sms / 2);
    if (log_enabled())
      std::fprintf(stderr, "dmuon: device %d: %d SMs, %d co-resident CTA pairs for the pair GEMM\n", dev,
                   d.sms, nc);
  }
  const void* pk[] = {reinterpret_cast<const void*>(&prologue_kernel<__nv_bfloat16, false>),
                      reinterpret_cast<const void*>(&prologue_kernel<float, false>),
                      reinterpret_cast<const void*>(&prologue_kernel<__nv_bfloat16, true>),
                      reinterpret_cast<const void*>(&prologue_kernel<float, true>)};
  for (const void* k : pk) {
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kProSmemBytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prologue smem)");
  }
  e = cudaFuncSetAttribute(reinterpret_cast<const void*>(&prologue_tma_kernel<true>),
                           cudaFuncAttributeMaxDynamicSharedMemorySize, PtCfg<true>::kSmem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(pipelined prologue smem)");
  e = cudaFuncSetAttribute(reinterpret_cast<const void*>(&prologue_tma_kernel<false>),
                           cudaFuncAttributeMaxDynamicSharedMemorySize, PtCfg<false>::kSmem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(pipelined prologue smem)");
  if (!encode_fn()) return fail(DMUON_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cudaMemPoolProps props;
  std::memset(&props, 0, sizeof(props));
  props.allocType = cudaMemAllocationTypePinned;
  props.location.type = cudaMemLocationTypeDevice;
  props.location.id = dev;
  e = cudaMemPoolCreate(&d.pool, &props);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemPoolCreate");
  uint64_t keep = UINT64_MAX;
  e = cudaMemPoolSetAttribute(d.pool, cudaMemPoolAttrReleaseThreshold, &keep);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemPoolSetAttribute");
  d.ready = true;
  return DMUON_OK;
}

int64_t g_plan_builds = 0;   // launch plans built in this process

// Writes `bytes` (a multiple of 16) of host data to device memory with
// upload kernels on `st`: stream ordered, no host staging, no synchronous copy.
void enqueue_upload(void* dst, const uint8_t* src, size_t bytes, cudaStream_t st) {
  std::unique_ptr<UploadParams> up(new UploadParams());
  const size_t words = bytes / 16;
  for (size_t w0 = 0; w0 < words; w0 += kUploadWords) {
    const int n = static_cast<int>(std::min<size_t>(kUploadWords, words - w0));
    up->dst = reinterpret_cast<uint4*>(dst) + w0;
    up->nwords = n;
    std::memcpy(up->w, src + w0 * 16, static_cast<size_t>(n) * 16);
    ++g_launches;
    upload_kernel<<<1, 256, 0, st>>>(*up);
  }
}

// Device pointers already checked (per device).  A checked address stays
// device memory: under unified addressing, host and device allocations never
// share virtual addresses.
std::unordered_set<const void*> g_checked[64];

// 0 when `p` is device (or managed) memory; DMUON_ERR_INVALID_ARG for host
// memory (page-locked or not); nothing is launched either way.
int classify_pointer(const void* p) {
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return DMUON_ERR_INVALID_ARG;
  }
  return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) ? DMUON_OK : DMUON_ERR_INVALID_ARG;
}

int check_device_ptr(int dev, const void* p, int i, const char* what, const char* kind = "matrix") {
  if (p == nullptr) return DMUON_OK;
  std::unordered_set<const void*>& seen = g_checked[dev];
  if (seen.count(p)) return DMUON_OK;
  if (classify_pointer(p) != DMUON_OK)
    return fail(DMUON_ERR_INVALID_ARG, "%s %d: %s is not device memory (host memory cannot be "
                "passed to the kernels)", kind, i, what);
  if (seen.size() >= 65536) seen.clear();
  seen.insert(p);
  return DMUON_OK;
}

// 128 x 256 tiles of an m x m Gram (the quintic plans' SYRK, whose A is
// mirrored, and the SQUARE stage): column bands of 256 with row bands
// 0..2J+1 of 128.
int64_t syrk_tiles_of(int64_t m) {
  const int64_t nJ = cdiv(m, kBN), nI = cdiv(m, kBM);
  return (nJ - 1) * nJ + nI;
}
// 256 x 256 upper tiles of an m x m Gram (syrk256_kernel).
int64_t syrk256_tiles_of(int64_t m) {
  const int64_t nJ = cdiv(m, kBN);
  return nJ * (nJ + 1) / 2;
}

// Which SYRK kernel a group runs.  A 256 x 256 tile does twice the work of a
// 128 x 256 tile in about 1.75 times its time (fewer operand bytes per FLOP),
// but a group with few tiles has fewer CTAs working: compare the waves of
// tiles over the SMs, each weighted by its tile time.  Small groups (the
// TinyMLP, one 256 x 512 matrix) keep the 128 x 256 tiles; a 4096 x 4096
// matrix (136 large tiles in one wave against 272 small ones in two) and the
// Llama-8B groups take the large ones.
bool use_syrk256(int64_t tiles128, int64_t tiles256, int sms) {
  const double w128 = static_cast<double>(cdiv(tiles128, sms));
  const double w256 = static_cast<double>(cdiv(tiles256, sms));
  return 1.75 * w256 < w128;
}
int64_t gemm_tiles_of(int64_t m, int64_t n) { return cdiv(m, kBM) * cdiv(n, kBN); }
// 256 x 256 tiles of the pair GEMM (gemm_pair_kernel).
int64_t gemm_pair_tiles_of(int64_t m, int64_t n) { return cdiv(m, 2 * kBM) * cdiv(n, kBN); }

// Builds (or finds) the plan for these matrices and this workspace.
// 16-byte vector access of a matrix's parameter, gradient and buffer rows.
int vec4_of(const MatIn& x) {
  bool v = (x.cols % 4 == 0) && aligned(x.W, 16) && aligned(x.G, 16) && (x.buf == nullptr || aligned(x.buf, 16));
  for (const void* q : x.gr) v = v && aligned(q, 16);
  return v ? 1 : 0;
}

PtrSet ptrs_of(const MatIn& x) {
  PtrSet p;
  p.W = x.W;
  p.G = x.G;
  p.buf = x.buf;
  p.vec4 = vec4_of(x);
  return p;
}

// Builds (or finds) the plan for these shapes and this workspace; a new
// plan's device memory is allocated from the pool and uploaded on `st`.
bool capturing(cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return cs != cudaStreamCaptureStatusNone;
}

int get_plan(const std::vector<MatIn>& in, int steps, bool quintic, void* ws, int dev, cudaStream_t st,
             Plan** out) {
  std::vector<uint8_t> key;
  key.reserve(64 + in.size() * 48);
  put(key, dev);
  put(key, steps > 1 ? 2 : steps);
  put(key, quintic);
  put(key, ws);
  put(key, static_cast<int64_t>(in.size()));
  for (const MatIn& x : in) {
    put(key, x.rows); put(key, x.cols);
    put(key, x.pdt); put(key, x.gdt); put(key, x.mode); put(key, x.lr_mult);
    put(key, static_cast<int64_t>(x.gr.size()));
    for (const void* q : x.gr) put(key, q);
  }
  const uint64_t h = fnv1a(key.data(), key.size());
  for (auto it = g_plans.begin(); it != g_plans.end(); ++it) {
    if ((*it)->hash == h && (*it)->key == key) {
      g_plans.splice(g_plans.begin(), g_plans, it);
      *out = g_plans.front().get();
      return DMUON_OK;
    }
  }

  if (capturing(st))
    // A plan's memory and upload must not belong to a graph: the shapes are
    // planned by an eager call first.
    return fail(DMUON_ERR_UNSUPPORTED, "these shapes have no launch plan yet and the stream is "
                "capturing a graph: make one call with them before the capture");
  const Layout L = make_layout(in, steps, quintic);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const int nmat = static_cast<int>(in.size());

  // Host image of the plan's device memory.
  std::vector<MatDesc> descs(nmat);
  std::vector<MatMaps> maps(nmat);
  struct GroupArrays {
    std::vector<int> so, sp, go, gp, qp;
    std::vector<int64_t> pp;
  };
  std::vector<GroupArrays> ga(L.groups.size());
  std::unique_ptr<Plan> P(new Plan());
  P->key = std::move(key);
  P->hash = h;
  P->device = dev;
  P->quintic = quintic;

  int first = 0;
  std::vector<int> desc_of(nmat, -1);
  for (size_t gi = 0; gi < L.groups.size(); ++gi) {
    const GroupLayout& g = L.groups[gi];
    const int dt = g.dtype;
    const int eb = elem_bytes(dt);
    const int BK = 128 / eb;
    GroupPlan gp{};
    gp.dtype = dt;
    gp.nmat = static_cast<int>(g.idx.size());
    gp.first = first;
    gp.ptiles = g.ptiles;
    GroupArrays& A = ga[gi];
    A.pp.push_back(0);
    {
      // The SYRK kernel, then the GEMM kernel: CTA pairs for bf16 groups on
      // 256 x 256 SYRK tiles whose matrices have n % 64 == 0 (3-D X operand
      // loads).  Any m: rows past m load as zeros and are not stored.
      int64_t t128 = 0, t256 = 0;
      bool pair_ok = dt == DMUON_BF16 && g_dev[dev].pair_clusters > 0;
      for (int k = 0; k < gp.nmat; ++k) {
        const MatLayout& ml = L.mats[g.idx[k]];
        t128 += syrk_tiles_of(ml.m);
        t256 += syrk256_tiles_of(ml.m);
        pair_ok = pair_ok && ml.n % 64 == 0;
      }
      gp.syrk256 = use_syrk256(t128, t256, g_dev[dev].sms);
      gp.gemm_pair = gp.syrk256 && pair_ok;
    }
    for (int k = 0; k < gp.nmat; ++k) {
      const int i = g.idx[k];
      const MatIn& x = in[i];
      const MatLayout& ml = L.mats[i];
      MatDesc& d = descs[first + k];
      desc_of[i] = first + k;
      std::memset(&d, 0, sizeof(d));
      d.W = x.W; d.G = x.G; d.buf = x.buf;
      d.rows = x.rows; d.cols = x.cols;
      d.ldx = ml.ldx; d.lda = ml.lda;
      d.X[0] = wsb + ml.x0;
      d.X[1] = (ml.x1 != SIZE_MAX) ? wsb + ml.x1 : nullptr;
      d.Xop[0] = wsb + ml.o0;
      d.Xop[1] = (ml.o1 != SIZE_MAX) ? wsb + ml.o1 : nullptr;
      d.A = (ml.a != SIZE_MAX) ? wsb + ml.a : nullptr;
      d.P = (ml.p != SIZE_MAX) ? wsb + ml.p : nullptr;
      d.scale = reinterpret_cast<float*>(wsb + g.scales) + k;
      d.lr_mult = x.lr_mult;
      d.m = static_cast<int>(ml.m); d.n = static_cast<int>(ml.n);
      d.T = x.rows > x.cols ? 1 : 0;
      d.mode = x.mode;
      d.g_bf16 = x.gdt == DMUON_BF16 ? 1 : 0;
      d.vec4 = vec4_of(x);
      d.world = x.gr.size() > 1 ? static_cast<int>(x.gr.size()) : 1;
      if (d.world > 1) gp.ranks = true;
      if (!d.g_bf16) gp.g_bf16 = false;
      d.Gr = nullptr;   // set once the plan's device memory exists
      d.ptiles_c = static_cast<int>(ml.ptiles_c);
      A.pp.push_back(A.pp.back() + ml.ptiles);
      if (ws) {
        MatMaps& mm = maps[first + k];
        std::memset(&mm, 0, sizeof(mm));
        bool okm = true;
        // 3-D MN-major maps when every buffer of the matrix allows them.
        d.b3d = (dt == DMUON_BF16 && ml.n % 64 == 0) ? 1 : 0;
        for (int b = 0; b < 2 && d.b3d; ++b)
          if (d.Xop[b] && !encode_mn3d(&mm.xmn[b], d.Xop[b], ml.n, ml.m, ml.ldx)) d.b3d = 0;
        for (int b = 0; b < 2; ++b) {
          void* xb = d.Xop[b];
          if (!xb) {
            mm.xk[b] = mm.xk[0]; mm.xkw[b] = mm.xkw[0]; mm.xmn[b] = mm.xmn[0]; mm.xmn2[b] = mm.xmn2[0];
            continue;
          }
          okm &= encode_2d(&mm.xk[b], dt, xb, ml.n, ml.m, ml.ldx, BK, kBM);
          okm &= encode_2d(&mm.xkw[b], dt, xb, ml.n, ml.m, ml.ldx, BK, kBN);
          // MN-major 32-bit operands need 32-byte swizzle units.
          if (!d.b3d)
            okm &= encode_2d(&mm.xmn[b], dt, xb, ml.n, ml.m, ml.ldx, BK, BK,
                             dt == DMUON_F32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B
                                             : CU_TENSOR_MAP_SWIZZLE_128B);
          if (gp.gemm_pair) okm &= d.b3d && encode_mn3d(&mm.xmn2[b], xb, ml.n, ml.m, ml.ldx, 2);
        }
        const CUtensorMapSwizzle mn_sw =
            dt == DMUON_F32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B;
        if (d.A) {
          okm &= encode_2d(&mm.a, dt, d.A, ml.m, ml.m, ml.lda, BK, kBM);
          okm &= encode_2d(&mm.amn, dt, d.A, ml.m, ml.m, ml.lda, BK, BK, mn_sw);
        }
        // A as a 3-D MN-major view: one load per transposed operand of the
        // quintic SQUARE stage.
        d.a3d = 0;
        if (d.P && dt == DMUON_BF16 && ml.m % 64 == 0)
          d.a3d = (encode_mn3d(&mm.amn3[0], d.A, ml.m, ml.m, ml.lda, 4) &&
                   encode_mn3d(&mm.amn3[1], d.A, ml.m, ml.m, ml.lda, 2)) ? 1 : 0;
        if (d.P) {
          okm &= encode_2d(&mm.aw, dt, d.A, ml.m, ml.m, ml.lda, BK, kBN);
          okm &= encode_2d(&mm.p, dt, d.P, ml.m, ml.m, ml.lda, BK, kBM);
          okm &= encode_2d(&mm.pmn, dt, d.P, ml.m, ml.m, ml.lda, BK, BK, mn_sw);
        }
        // Transposed bf16 matrices with 16-byte aligned rows: the prologue
        // loads each 64 x 128 item of G and buf with one 2-D tensor load.
        // The maps hold the caller's addresses (a placeholder in the
        // workspace while they are not 16-byte aligned); patch_kernel keeps
        // them current.
        d.tmaps = 0;
        if (d.T && dt == DMUON_BF16 && d.world <= 1 && x.cols % 8 == 0) {
          const bool ga = aligned(x.G, 16), ba = x.buf == nullptr || aligned(x.buf, 16);
          void* gbase = ga ? const_cast<void*>(x.G) : static_cast<void*>(wsb);
          void* bbase = (x.buf && ba) ? static_cast<void*>(x.buf) : static_cast<void*>(wsb);
          bool okt = encode_2d(&mm.gt, x.gdt, gbase, x.cols, x.rows, x.cols, kTC, kTR,
                               CU_TENSOR_MAP_SWIZZLE_NONE);
          if (x.buf) okt = okt && encode_2d(&mm.bt, DMUON_F32, bbase, x.cols, x.rows, x.cols, kTC, kTR,
                                            CU_TENSOR_MAP_SWIZZLE_NONE);
          d.tmaps = okt ? 1 : 0;
        }
        if (!okm) return fail(DMUON_ERR_CUDA, "cuTensorMapEncodeTiled failed for matrix %d", i);
      }
    }
    // Longest K first: SYRK contracts over n, the GEMM over m.
    std::vector<int> ord(gp.nmat);
    for (int k = 0; k < gp.nmat; ++k) ord[k] = k;
    std::vector<int> so = ord, go = ord;
    std::stable_sort(so.begin(), so.end(), [&](int a, int b) {
      const MatDesc& x = descs[first + a]; const MatDesc& y = descs[first + b];
      return x.n != y.n ? x.n > y.n : x.m > y.m;
    });
    std::stable_sort(go.begin(), go.end(), [&](int a, int b) {
      const MatDesc& x = descs[first + a]; const MatDesc& y = descs[first + b];
      return x.m != y.m ? x.m > y.m : x.n > y.n;
    });
    gp.square256 = gp.gemm_pair;
    for (int k = 0; k < gp.nmat; ++k) gp.square256 = gp.square256 && descs[first + k].a3d;
    int64_t st = 0, gt = 0, qt = 0;
    A.sp.push_back(0);
    A.gp.push_back(0);
    A.qp.push_back(0);
    for (int k = 0; k < gp.nmat; ++k) {
      const int64_t mk = descs[first + so[k]].m;
      st += gp.syrk256 ? syrk256_tiles_of(mk) : syrk_tiles_of(mk);
      gt += gp.gemm_pair ? gemm_pair_tiles_of(descs[first + go[k]].m, descs[first + go[k]].n)
                         : gemm_tiles_of(descs[first + go[k]].m, descs[first + go[k]].n);
      // SQUARE contracts over m, in the GEMM's order; on 256 x 256 tiles
      // (syrk256_kernel) when square256, else on 128 x 256 ones
      qt += gp.square256 ? syrk256_tiles_of(descs[first + go[k]].m) : syrk_tiles_of(descs[first + go[k]].m);
      A.sp.push_back(static_cast<int>(st));
      A.gp.push_back(static_cast<int>(gt));
      A.qp.push_back(static_cast<int>(qt));
    }
    if (st > INT32_MAX || gt > INT32_MAX)
      return fail(DMUON_ERR_UNSUPPORTED, "too many tiles in one launch");
    A.so = so; A.go = go;
    gp.syrk_tiles = static_cast<int>(st);
    gp.gemm_tiles = static_cast<int>(gt);
    gp.square_tiles = static_cast<int>(qt);
    gp.partials = reinterpret_cast<float*>(wsb + g.partials);
    gp.gpartials = reinterpret_cast<double*>(wsb + g.gpartials);
    P->groups.push_back(gp);
    first += gp.nmat;
  }

  // Pack: descs | maps | per group (pprefix, syrk order/prefix, gemm order/prefix).
  size_t off = 0;
  const size_t o_desc = off; off = align_up(off + sizeof(MatDesc) * nmat, 128);
  const size_t o_maps = off; off = align_up(off + sizeof(MatMaps) * nmat, 128);
  constexpr int kArr = 6;
  std::vector<size_t> o_g(ga.size() * kArr);
  for (size_t gi = 0; gi < ga.size(); ++gi) {
    o_g[gi * kArr + 0] = off; off = align_up(off + sizeof(int64_t) * ga[gi].pp.size(), 128);
    o_g[gi * kArr + 1] = off; off = align_up(off + sizeof(int) * ga[gi].so.size(), 128);
    o_g[gi * kArr + 2] = off; off = align_up(off + sizeof(int) * ga[gi].sp.size(), 128);
    o_g[gi * kArr + 3] = off; off = align_up(off + sizeof(int) * ga[gi].go.size(), 128);
    o_g[gi * kArr + 4] = off; off = align_up(off + sizeof(int) * ga[gi].gp.size(), 128);
    o_g[gi * kArr + 5] = off; off = align_up(off + sizeof(int) * ga[gi].qp.size(), 128);
  }
  // The ranks' gradient buffers of matrices that average several (rank order).
  std::vector<const void*> gr_ptrs;
  std::vector<int64_t> gr_at(nmat, -1);
  for (int i = 0; i < nmat; ++i) {
    if (in[i].gr.size() > 1) {
      gr_at[desc_of[i]] = static_cast<int64_t>(gr_ptrs.size());
      gr_ptrs.insert(gr_ptrs.end(), in[i].gr.begin(), in[i].gr.end());
    }
  }
  const size_t o_gr = off; off = align_up(off + sizeof(void*) * gr_ptrs.size(), 128);
  cudaError_t e = cudaEventCreateWithFlags(&P->last, cudaEventDisableTiming);
  if (e != cudaSuccess) {
    P->last = nullptr;
    return cuda_fail(e, "cudaEventCreate");
  }
  e = lib_malloc_async(&P->dmem, off, g_dev[dev].pool, st);
  if (e != cudaSuccess) {
    P->dmem = nullptr;
    cudaGetLastError();
    return fail(DMUON_ERR_NO_WORKSPACE, "plan allocation of %zu bytes failed", off);
  }
  uint8_t* base = static_cast<uint8_t*>(P->dmem);
  for (int k = 0; k < nmat; ++k)
    if (gr_at[k] >= 0)
      descs[k].Gr = reinterpret_cast<const void* const*>(base + o_gr + sizeof(void*) * gr_at[k]);
  std::vector<uint8_t> img(off, 0);
  if (!gr_ptrs.empty()) std::memcpy(img.data() + o_gr, gr_ptrs.data(), sizeof(void*) * gr_ptrs.size());
  std::memcpy(img.data() + o_desc, descs.data(), sizeof(MatDesc) * nmat);
  std::memcpy(img.data() + o_maps, maps.data(), sizeof(MatMaps) * nmat);
  for (size_t gi = 0; gi < ga.size(); ++gi) {
    std::memcpy(img.data() + o_g[gi * kArr + 0], ga[gi].pp.data(), sizeof(int64_t) * ga[gi].pp.size());
    std::memcpy(img.data() + o_g[gi * kArr + 1], ga[gi].so.data(), sizeof(int) * ga[gi].so.size());
    std::memcpy(img.data() + o_g[gi * kArr + 2], ga[gi].sp.data(), sizeof(int) * ga[gi].sp.size());
    std::memcpy(img.data() + o_g[gi * kArr + 3], ga[gi].go.data(), sizeof(int) * ga[gi].go.size());
    std::memcpy(img.data() + o_g[gi * kArr + 4], ga[gi].gp.data(), sizeof(int) * ga[gi].gp.size());
    std::memcpy(img.data() + o_g[gi * kArr + 5], ga[gi].qp.data(), sizeof(int) * ga[gi].qp.size());
  }
  enqueue_upload(P->dmem, img.data(), img.size(), st);
  e = cudaEventRecord(P->last, st);
  if (e != cudaSuccess) return cuda_fail(e, "plan upload");
  P->last_st = st;
  ++g_plan_builds;
  P->desc_of = desc_of;
  P->cur.resize(nmat);
  for (int i = 0; i < nmat; ++i) P->cur[desc_of[i]] = ptrs_of(in[i]);
  for (size_t gi = 0; gi < P->groups.size(); ++gi) {
    GroupPlan& gp = P->groups[gi];
    gp.pprefix = reinterpret_cast<const int64_t*>(base + o_g[gi * kArr + 0]);
    gp.syrk_order = reinterpret_cast<const int*>(base + o_g[gi * kArr + 1]);
    gp.syrk_prefix = reinterpret_cast<const int*>(base + o_g[gi * kArr + 2]);
    gp.gemm_order = reinterpret_cast<const int*>(base + o_g[gi * kArr + 3]);
    gp.gemm_prefix = reinterpret_cast<const int*>(base + o_g[gi * kArr + 4]);
    gp.square_prefix = reinterpret_cast<const int*>(base + o_g[gi * kArr + 5]);
  }
  P->clip = reinterpret_cast<float*>(wsb + L.clip);
  P->d_mats = reinterpret_cast<const MatDesc*>(base + o_desc);
  P->d_maps = reinterpret_cast<const MatMaps*>(base + o_maps);
  if (log_enabled()) {
    int64_t syrk = 0, gemm = 0, items = 0;
    for (const GroupPlan& gp : P->groups) { syrk += gp.syrk_tiles; gemm += gp.gemm_tiles; items += gp.ptiles; }
    std::fprintf(stderr, "dmuon: plan on device %d: %d matrices in %zu dtype groups, %lld prologue items, "
                 "%lld SYRK and %lld GEMM tiles per stage, scratch %zu bytes, plan %zu bytes\n", dev, nmat,
                 P->groups.size(), static_cast<long long>(items), static_cast<long long>(syrk),
                 static_cast<long long>(gemm), L.bytes, img.size());
  }
  g_plans.emplace_front(std::move(P));
  Plan* plan = g_plans.front().get();
  while (g_plans.size() > kMaxPlans) {
    // An evicted plan may still be read by queued kernels: its memory is
    // freed in stream order after the latest work that used it.
    Plan& old = *g_plans.back();
    if (old.dmem) {
      free_in_order(old.dmem, st, old.last);
      old.dmem = nullptr;
    }
    g_plans.pop_back();
  }
  *out = plan;
  return DMUON_OK;
}

// Launches `kernel` on `st` with programmatic stream serialization: its CTAs
// may be scheduled while the previous kernel in the stream is still running.
// Every library kernel begins with griddep_wait(), so none touches memory
// before that kernel has completed; what overlaps is the launch and CTA
// dispatch.  Errors surface as for a <<<>>> launch (cudaGetLastError).
template <typename... KArgs, typename... Args>
void launch_pdl(void (*kernel)(KArgs...), int grid, int block, size_t smem, cudaStream_t st,
                Args&&... args) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(block));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr;
  std::memset(&attr, 0, sizeof(attr));
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Before a plan's kernels run on `st`: order after the plan's latest use on
// another stream, then write the caller's addresses where they differ from
// the ones the descriptors hold.
//
// While `st` captures a graph, every address is patched (so that each replay
// writes the addresses it was captured with, whatever eager calls did in
// between), and from then on every call on the plan patches every address: a
// replay may rewrite them at any time, so the host's record is no longer the
// device's.  The ordering against other streams is the graph's, so no event
// is waited on or recorded during capture.
int prepare_plan(Plan& P, const std::vector<MatIn>& in, cudaStream_t st) {
  const bool cap = capturing(st);
  cudaError_t e = cudaSuccess;
  if (!cap && P.last_st != st) e = cudaStreamWaitEvent(st, P.last, 0);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  std::unique_ptr<PatchParams> pp;
  auto flush = [&]() {
    if (!pp || pp->n == 0) return;
    ++g_launches;
    launch_pdl(patch_kernel, 1, 256, 0, st, *pp);
    pp->n = 0;
  };
  for (size_t i = 0; i < in.size(); ++i) {
    const int d = P.desc_of[i];
    const PtrSet now = ptrs_of(in[i]);
    if (!cap && !P.captured && now == P.cur[d]) continue;
    if (!pp) {
      pp.reset(new PatchParams());
      pp->mats = const_cast<MatDesc*>(P.d_mats);
      pp->maps = const_cast<MatMaps*>(P.d_maps);
      pp->n = 0;
    }
    PatchEntry& en = pp->e[pp->n++];
    en.W = now.W;
    en.G = now.G;
    en.buf = now.buf;
    en.index = d;
    en.vec4 = now.vec4;
    P.cur[d] = now;
    if (pp->n == kPatchMax) flush();
  }
  flush();
  if (cap) P.captured = true;
  return DMUON_OK;
}

// After a plan's kernels were enqueued on `st`.
int finish_plan(Plan& P, cudaStream_t st) {
  if (capturing(st)) return DMUON_OK;
  cudaError_t e = cudaEventRecord(P.last, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  P.last_st = st;
  return DMUON_OK;
}

// ------------------------------------------------------------------ launch
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per bounded device wait

// Launch bookkeeping: a process-wide launch counter (g_launches, above) and,
// when enabled, CUDA-event brackets around each launch for per-kernel device time.
bool g_timing = false;
struct Bracket {
  cudaEvent_t a, b;
  int kind;
  bool own_a;     // a is this bracket's own event (not the previous bracket's b)
};
std::vector<Bracket> g_brackets;       // recorded, not yet harvested
std::vector<cudaEvent_t> g_event_pool;
double g_kind_ms[DMUON_KERNEL_KINDS] = {0};
int64_t g_kind_n[DMUON_KERNEL_KINDS] = {0};

cudaEvent_t pool_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// NVTX range names of the kernel kinds (a timeline tool shows every launch;
// without one attached the calls cost next to nothing).
const char* const kKindNames[DMUON_KERNEL_KINDS] = {"dmuon prologue", "dmuon finalize", "dmuon syrk",
                                                    "dmuon gemm",     "dmuon apply",    "dmuon adamw",
                                                    "dmuon clip",     "dmuon square"};

// Inside a TimingChain (one group's launches, back to back on one stream,
// nothing else enqueued between them) a bracket starts at the previous
// bracket's end event: one event per launch instead of two.
bool g_chain_active = false;
cudaEvent_t g_chain_event = nullptr;
cudaStream_t g_chain_stream = nullptr;
struct TimingChain {
  TimingChain() { g_chain_active = true; g_chain_event = nullptr; }
  ~TimingChain() { g_chain_active = false; g_chain_event = nullptr; }
};

struct LaunchScope {
  cudaStream_t st;
  int kind;
  cudaEvent_t a = nullptr;
  bool own_a = true;
  LaunchScope(cudaStream_t s, int k) : st(s), kind(k) {
    ++g_launches;
    nvtxRangePushA(kKindNames[k]);
    if (g_timing) {
      if (g_chain_active && g_chain_event && g_chain_stream == st) {
        a = g_chain_event;
        own_a = false;
      } else {
        a = pool_event();
        cudaEventRecord(a, st);
      }
    }
  }
  ~LaunchScope() {
    if (a) {
      cudaEvent_t b = pool_event();
      cudaEventRecord(b, st);
      g_brackets.push_back(Bracket{a, b, kind, own_a});
      if (g_chain_active) {
        g_chain_event = b;
        g_chain_stream = st;
      }
    }
    nvtxRangePop();
  }
};

// One Newton-Schulz stage over all tiles of a group: a persistent grid of at
// most one CTA per SM.
template <int kMode, typename E>
void launch_ns_stage(const NsParams& np, const DeviceInfo& d, cudaStream_t st) {
  launch_pdl(ns_stage_kernel<kMode, E>, std::min(np.ntiles, d.sms), kNsThreads, kNsSmemBytes, st, np);
}

template <typename E>
ElemParams elem_params(const Plan& P, const GroupPlan& g, const StepOpts& o) {
  ElemParams ep;
  ep.mats = P.d_mats + g.first;
  ep.ptile_prefix = g.pprefix;
  ep.partials = g.partials;
  ep.nmat = g.nmat;
  ep.ntiles = g.ptiles;
  ep.mu = o.mu;
  ep.nesterov = o.nesterov;
  ep.lr = o.lr;
  ep.wd = o.wd;
  ep.clip = o.max_norm > 0.0f ? P.clip : nullptr;
  ep.gpartials = g.gpartials;
  ep.err = nullptr;
  ep.wait_limit_ns = 0;
  ep.maps = P.d_maps + g.first;
  return ep;
}

template <typename E>
void launch_grad_norm(const Plan& P, const GroupPlan& g, const DeviceInfo& d, const StepOpts& o,
                      cudaStream_t st) {
  const ElemParams ep = elem_params<E>(P, g, o);
  const int pgrid = static_cast<int>(std::min<int64_t>(g.ptiles, static_cast<int64_t>(d.sms) * 8));
  LaunchScope ls(st, DMUON_KERNEL_PROLOGUE);
  if (g.ranks) launch_pdl(grad_norm_kernel<E, true>, pgrid, kPThreads, 0, st, ep);
  else launch_pdl(grad_norm_kernel<E, false>, pgrid, kPThreads, 0, st, ep);
}

template <typename E>
void launch_group(const Plan& P, const GroupPlan& g, const DeviceInfo& d, const StepOpts& o,
                  cudaStream_t st) {
  const float lr = o.lr, wd = o.wd;
  const int steps = o.steps;
  TimingChain chain;   // the group's launches follow one another on `st`
  ElemParams ep = elem_params<E>(P, g, o);
  ep.err = d.err;
  ep.wait_limit_ns = kWaitLimitNs;
  const int pgrid = static_cast<int>(std::min<int64_t>(g.ptiles, static_cast<int64_t>(d.sms) * 8));
  {
    LaunchScope ls(st, DMUON_KERNEL_PROLOGUE);
    if (g.ranks) {
      launch_pdl(prologue_kernel<E, true>, pgrid, kPThreads, kProSmemBytes, st, ep);
    } else if (sizeof(E) == 2) {
      // bf16 iterates: the pipelined prologue, two blocks per SM when every
      // gradient is bf16 (48 KB stages), else one (64 KB stages).
      const int per_sm = g.g_bf16 ? PtCfg<true>::kBlocksPerSm : PtCfg<false>::kBlocksPerSm;
      const int tgrid = static_cast<int>(std::min<int64_t>(g.ptiles, static_cast<int64_t>(d.sms) * per_sm));
      if (g.g_bf16) launch_pdl(prologue_tma_kernel<true>, tgrid, kPtThreads, PtCfg<true>::kSmem, st, ep);
      else launch_pdl(prologue_tma_kernel<false>, tgrid, kPtThreads, PtCfg<false>::kSmem, st, ep);
    } else {
      launch_pdl(prologue_kernel<E, false>, pgrid, kPThreads, kProSmemBytes, st, ep);
    }
  }
  {
    LaunchScope ls(st, DMUON_KERNEL_FINALIZE);
    launch_pdl(finalize_kernel, g.nmat, 32, 0, st, ep);
  }
  if (steps == 0) {
    LaunchScope ls(st, DMUON_KERNEL_APPLY);
    launch_pdl(apply_kernel<E>, pgrid, kPThreads, 0, st, ep);
    return;
  }
  NsParams np;
  np.mats = P.d_mats + g.first;
  np.maps = P.d_maps + g.first;
  np.nmat = g.nmat;
  np.lr = lr;
  np.wd = wd;
  np.quintic = P.quintic ? 1 : 0;
  // The quintic SQUARE stage reads all of A: mirrored by the SYRK, or, on pair
  // groups (whose A holds whole diagonal 256-blocks), read from the upper
  // triangle with the lower k-blocks transposed.
  np.mirror = (P.quintic && !g.gemm_pair) ? 1 : 0;
  np.a_upper = 1;                    // the GEMM reads A (or P) from its upper triangle
  np.diag_full = g.gemm_pair ? 1 : 0;  // the pair GEMM reads whole diagonal 256-blocks
  np.ca = o.ca;
  np.cb = P.quintic ? 1.0f : o.cb;   // quintic: X <- a X + P X with P = b A + c A A
  np.cc = 0.0f;
  np.err = d.err;
  np.wait_limit_ns = kWaitLimitNs;
  for (int s = 0; s < steps; ++s) {
    np.cur = s & 1;
    np.first = s == 0;
    np.last = s == steps - 1;
    np.order = g.syrk_order;
    np.tile_prefix = g.syrk_prefix;
    np.ntiles = g.syrk_tiles;
    {
      LaunchScope ls(st, DMUON_KERNEL_SYRK);
      if (g.syrk256) launch_pdl(syrk256_kernel<E>, std::min(np.ntiles, d.sms), kNsThreads, kS2SmemBytes, st, np);
      else launch_ns_stage<kSyrk, E>(np, d, st);
    }
    if (P.quintic) {
      NsParams sq = np;
      sq.cb = o.cb;
      sq.cc = o.cc;
      sq.mirror = 0;
      sq.a_upper = g.gemm_pair ? 1 : 0;
      sq.diag_full = g.gemm_pair ? 1 : 0;   // the pair GEMM reads P's whole diagonal 256-blocks
      sq.order = g.gemm_order;
      sq.tile_prefix = g.square_prefix;
      sq.ntiles = g.square_tiles;
      LaunchScope ls(st, DMUON_KERNEL_SQUARE);
      bool big = false;
      if constexpr (sizeof(E) == 2) {
        if (g.square256) {
          // 256 x 256 tiles; A holds its upper triangle and whole diagonal 256-blocks
          launch_pdl(syrk256_kernel<E, kSquare>, std::min(sq.ntiles, d.sms), kNsThreads, kS2SmemBytes, st, sq);
          big = true;
        }
      }
      if (!big) launch_ns_stage<kSquare, E>(sq, d, st);
    }
    np.order = g.gemm_order;
    np.tile_prefix = g.gemm_prefix;
    np.ntiles = g.gemm_tiles;
    {
      LaunchScope ls(st, DMUON_KERNEL_GEMM);
      if (g.gemm_pair)
        launch_pdl(gemm_pair_kernel, 2 * std::min(np.ntiles, d.pair_clusters), kNsThreads, kG2SmemBytes, st, np);
      else
        launch_ns_stage<kGemm, E>(np, d, st);
    }
  }
}

int launch_plan(const Plan& P, const StepOpts& o, cudaStream_t st) {
  const DeviceInfo& d = g_dev[P.device];
  if (o.max_norm > 0.0f) {
    // Global gradient norm over every matrix of the call, then the clip
    // coefficient that the prologues apply.
    ClipParams cp;
    cp.part[0] = cp.part[1] = nullptr;
    cp.count[0] = cp.count[1] = 0;
    for (size_t gi = 0; gi < P.groups.size() && gi < 2; ++gi) {
      const GroupPlan& g = P.groups[gi];
      if (g.dtype == DMUON_BF16) launch_grad_norm<__nv_bfloat16>(P, g, d, o, st);
      else launch_grad_norm<float>(P, g, d, o, st);
      cp.part[gi] = g.gpartials;
      cp.count[gi] = g.ptiles;
    }
    cp.max_norm = o.max_norm;
    cp.coef = P.clip;
    cp.norm_out = o.norm_out;
    LaunchScope ls(st, DMUON_KERNEL_FINALIZE);
    launch_pdl(clip_coef_kernel, 1, 256, 0, st, cp);
  }
  for (const GroupPlan& g : P.groups) {
    if (g.dtype == DMUON_BF16) launch_group<__nv_bfloat16>(P, g, d, o, st);
    else launch_group<float>(P, g, d, o, st);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return DMUON_OK;
}

std::mutex g_api_mu;

int current_device(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  return device_setup(*dev);
}

// The library's scratch for calls on `st` that bring none: grown in stream
// order (the old region is freed after the work queued on `st` before it).
int arena_get(int dev, cudaStream_t st, size_t bytes, void** out) {
  Arena& a = g_arenas[std::make_pair(dev, st)];
  if (a.bytes < bytes && capturing(st))
    return fail(DMUON_ERR_UNSUPPORTED, "the stream's scratch arena must grow and the stream is "
                "capturing a graph: make one call with these shapes before the capture");
  if (a.bytes < bytes) {
    if (a.ptr) {
      free_in_order(a.ptr, st);
      a.ptr = nullptr;
      a.bytes = 0;
    }
    cudaError_t e = lib_malloc_async(&a.ptr, bytes, g_dev[dev].pool, st);
    if (e != cudaSuccess) {
      a.ptr = nullptr;
      cudaGetLastError();
      return fail(DMUON_ERR_NO_WORKSPACE, "scratch allocation of %zu bytes failed", bytes);
    }
    a.bytes = bytes;
  }
  *out = a.ptr;
  return DMUON_OK;
}

int gather(void* const params[], const void* const grads[], float* const bufs[],
           const dmuon_shape shapes[], int count, int ns_steps, int lr_scale,
           std::vector<MatIn>* in) {
  if (count < 0) return fail(DMUON_ERR_INVALID_ARG, "count must be >= 0");
  if (ns_steps < 0 || ns_steps > DMUON_MAX_STEPS)
    return fail(DMUON_ERR_INVALID_ARG, "ns_steps must be in [0, %d]", DMUON_MAX_STEPS);
  if (count == 0) return DMUON_OK;
  if (!params || !grads || !bufs || !shapes)
    return fail(DMUON_ERR_INVALID_ARG, "NULL array argument");
  in->reserve(count);
  for (int i = 0; i < count; ++i) {
    if (grads[i] == nullptr) continue;   // no gradient: skipped
    MatIn x;
    x.W = params[i];
    x.G = grads[i];
    x.buf = bufs[i];
    x.rows = shapes[i].rows;
    x.cols = shapes[i].cols;
    x.pdt = shapes[i].param_dtype;
    x.gdt = shapes[i].grad_dtype;
    x.mode = kModeMuon;
    x.lr_mult = 1.0f;
    if (lr_scale == DMUON_LR_SQRT_MAX)
      x.lr_mult = static_cast<float>(0.2 * std::sqrt(static_cast<double>(std::max(x.rows, x.cols))));
    const int r = check_matrix(x, i);
    if (r != DMUON_OK) return r;
    in->push_back(x);
  }
  return DMUON_OK;
}

// A large call runs as consecutive groups of matrices, one after the other on
// the stream, sharing one scratch region.  Measured on the Llama-8B stack
// (224 matrices, 7e9 elements): groups of one to four layers run at a higher
// SM clock under the power cap than one launch per stage over every matrix
// (413 ms against 440 ms per step).  With the current kernels, groups of
// about one layer (2^28 elements) run 0.5-2 % faster than two-layer groups
// and 3-4 % faster than four-layer ones, at a higher SM clock; the arithmetic
// of each matrix does not depend on the grouping.
constexpr int64_t kGroupElems = int64_t(1) << 28;
constexpr int kMaxGroups = 32;   // < kMaxPlans: one call never evicts its own plans

// Boundaries of consecutive groups: a matrix joins the current group unless
// that would take it past `target` elements.
std::vector<int> group_bounds(const std::vector<MatIn>& in, int64_t target) {
  std::vector<int> bnd(1, 0);
  int64_t acc = 0;
  for (size_t i = 0; i < in.size(); ++i) {
    const int64_t e = in[i].rows * in[i].cols;
    if (acc > 0 && acc + e > target) {
      bnd.push_back(static_cast<int>(i));
      acc = 0;
    }
    acc += e;
  }
  bnd.push_back(static_cast<int>(in.size()));
  return bnd;
}

// The groups of one call.  Clipping needs one global norm before any
// momentum update: one group.
std::vector<int> step_groups(const std::vector<MatIn>& in, bool clipping) {
  if (clipping) return {0, static_cast<int>(in.size())};
  int64_t total = 0;
  for (const MatIn& x : in) total += x.rows * x.cols;
  int64_t target = std::max<int64_t>(kGroupElems, (total + kMaxGroups - 1) / kMaxGroups);
  std::vector<int> bnd = group_bounds(in, target);
  while (static_cast<int>(bnd.size()) - 1 > kMaxGroups) {   // ends: target >= total gives one group
    target *= 2;
    bnd = group_bounds(in, target);
  }
  return bnd;
}

// Every tensor address of a call must be device memory: checked on the host
// before anything is enqueued (a kernel given host memory would fault).
int check_call_pointers(int dev, const std::vector<MatIn>& in) {
  for (size_t i = 0; i < in.size(); ++i) {
    const MatIn& x = in[i];
    int r = check_device_ptr(dev, x.W, static_cast<int>(i), x.mode == kModeMuon ? "the parameter" : "X");
    if (r == DMUON_OK && x.G != x.W) r = check_device_ptr(dev, x.G, static_cast<int>(i), "the gradient");
    if (r == DMUON_OK) r = check_device_ptr(dev, x.buf, static_cast<int>(i), "the momentum buffer");
    for (size_t q = 0; q < x.gr.size() && r == DMUON_OK; ++q)
      r = check_device_ptr(dev, x.gr[q], static_cast<int>(i), "a rank's gradient");
    if (r != DMUON_OK) return r;
  }
  return DMUON_OK;
}

int run(const std::vector<MatIn>& in, void* ws, size_t ws_bytes, bool own_ws, const StepOpts& o,
        cudaStream_t st) {
  const int steps = o.steps;
  if (in.empty()) return DMUON_OK;
  std::lock_guard<std::mutex> lk(g_api_mu);
  int dev = 0;
  int r = current_device(&dev);
  if (r != DMUON_OK) return r;
  r = check_call_pointers(dev, in);
  if (r != DMUON_OK) return r;
  const std::vector<int> bnd = step_groups(in, o.max_norm > 0.0f);
  const int ng = static_cast<int>(bnd.size()) - 1;
  std::vector<std::vector<MatIn>> sub(ng);
  size_t need = 0;
  for (int gi = 0; gi < ng; ++gi) {
    sub[gi].assign(in.begin() + bnd[gi], in.begin() + bnd[gi + 1]);
    need = std::max(need, make_layout(sub[gi], steps, o.cc != 0.0f).bytes);
  }
  if (own_ws) {
    r = arena_get(dev, st, need, &ws);
    if (r != DMUON_OK) return r;
  } else {
    if (!ws) return fail(DMUON_ERR_INVALID_ARG, "NULL workspace");
    if (ws_bytes < need)
      return fail(DMUON_ERR_NO_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed",
                  ws_bytes, need);
    if (!aligned(ws, 256)) return fail(DMUON_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    r = check_device_ptr(dev, ws, 0, "the workspace", "argument");
    if (r != DMUON_OK) return r;
  }
  // Every group's plan before any kernel of the call is enqueued (a new
  // plan's upload writes library memory only).  Groups with the same shapes
  // share one plan; its descriptors are patched with each group's addresses
  // in stream order.
  std::vector<Plan*> plans(ng, nullptr);
  for (int gi = 0; gi < ng; ++gi) {
    r = get_plan(sub[gi], steps, o.cc != 0.0f, ws, dev, st, &plans[gi]);
    if (r != DMUON_OK) return r;
  }
  for (int gi = 0; gi < ng; ++gi) {
    r = prepare_plan(*plans[gi], sub[gi], st);
    if (r == DMUON_OK) r = launch_plan(*plans[gi], o, st);
    if (r == DMUON_OK) r = finish_plan(*plans[gi], st);
    if (r != DMUON_OK) return r;
  }
  return DMUON_OK;
}

int check_opts(const StepOpts& o) {
  if (!std::isfinite(o.lr) || !std::isfinite(o.mu) || !std::isfinite(o.wd) || !std::isfinite(o.ca) ||
      !std::isfinite(o.cb) || !std::isfinite(o.cc))
    return fail(DMUON_ERR_INVALID_ARG, "lr, momentum, weight_decay and the NS coefficients must be finite");
  if (!(o.max_norm >= 0.0f) || !std::isfinite(o.max_norm))
    return fail(DMUON_ERR_INVALID_ARG, "max_grad_norm must be finite and >= 0");
  if (o.lr_scale != DMUON_LR_PLAIN && o.lr_scale != DMUON_LR_SQRT_MAX)
    return fail(DMUON_ERR_INVALID_ARG, "unknown lr_scale %d", o.lr_scale);
  return DMUON_OK;
}

StepOpts plain_opts(float lr, float momentum, int nesterov, float wd, int steps) {
  StepOpts o;
  o.lr = lr;
  o.mu = momentum;
  o.nesterov = nesterov ? 1 : 0;
  o.wd = wd;
  o.steps = steps;
  return o;
}

// ------------------------------------------------------------------ host-buffer step
// Two copy streams (upload, download) and a fixed set of events per device,
// created on the device's first host-buffer call and kept.  Events are
// re-recorded by later calls: a stream wait binds to the record that precedes
// it, so reuse is safe.
struct CopyLanes {
  bool ready = false;
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t ev[2 * DMUON_MAX_CHUNKS + 1] = {};
};
CopyLanes g_lanes[64];

int copy_lanes(int dev, CopyLanes** out) {
  CopyLanes& L = g_lanes[dev];
  if (!L.ready) {
    cudaError_t e = cudaStreamCreateWithFlags(&L.up, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&L.down, cudaStreamNonBlocking);
    for (cudaEvent_t& ev : L.ev)
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "copy stream set-up");
    L.ready = true;
  }
  *out = &L;
  return DMUON_OK;
}

bool page_locked(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

// Cut [0, n) into at most `chunks` runs of about equal `bytes`; returns the
// run boundaries (first 0, last n).
std::vector<int> chunk_bounds(const std::vector<size_t>& bytes, int chunks) {
  const int n = static_cast<int>(bytes.size());
  size_t total = 0;
  for (size_t b : bytes) total += b;
  std::vector<int> bnd(1, 0);
  size_t acc = 0;
  int c = 1;
  for (int i = 0; i + 1 < n; ++i) {
    acc += bytes[i];
    if (c < chunks && static_cast<double>(acc) * chunks >= static_cast<double>(total) * c) {
      bnd.push_back(i + 1);
      while (c < chunks && static_cast<double>(acc) * chunks >= static_cast<double>(total) * c) ++c;
    }
  }
  bnd.push_back(n);
  return bnd;
}

constexpr size_t kChunkTargetBytes = size_t(64) << 20;

// Automatic groups of the host-buffer step, by gradient bytes: the first
// group is small (its upload is exposed), each next one up to 1.5x the one
// before (an upload must land before the kernels reach it; the copy engines
// move ~55 GB/s, the update consumes gradients at ~35 GB/s), at most
// `mid` bytes (about the compute grouping of bf16 gradients), and the groups
// shrink again towards the end (the last
// group's download is exposed): a group may hold at most a third of the
// bytes still to come including itself.  At most DMUON_MAX_CHUNKS groups.
std::vector<int> ramp_bounds(const std::vector<size_t>& bytes) {
  const int n = static_cast<int>(bytes.size());
  size_t total = 0;
  for (size_t b : bytes) total += b;
  const size_t first = kChunkTargetBytes;
  const size_t mid = std::max(size_t(1) << 30, total / (DMUON_MAX_CHUNKS / 2));
  std::vector<int> bnd(1, 0);
  size_t acc = 0, done = 0;
  double grow = static_cast<double>(first);
  for (int i = 0; i + 1 < n; ++i) {
    acc += bytes[i];
    double target = std::min(static_cast<double>(mid), grow);
    target = std::min(target, std::max(static_cast<double>(first), static_cast<double>(total - done) / 3.0));
    if (static_cast<double>(acc) >= target && static_cast<int>(bnd.size()) < DMUON_MAX_CHUNKS) {
      bnd.push_back(i + 1);
      done += acc;
      acc = 0;
      grow *= 1.5;
    }
  }
  bnd.push_back(n);
  return bnd;
}

// in[k] are the matrices with a gradient; hg/hp/stage are parallel to in.
int run_host(const std::vector<MatIn>& in, const std::vector<const void*>& hg,
             const std::vector<void*>& hp, const std::vector<void*>& stage, int chunks, void* ws,
             size_t ws_bytes, bool own_ws, const StepOpts& o, cudaStream_t st) {
  if (in.empty()) return DMUON_OK;
  std::lock_guard<std::mutex> lk(g_api_mu);
  int dev = 0;
  int r = current_device(&dev);
  if (r != DMUON_OK) return r;
  r = check_call_pointers(dev, in);
  if (r != DMUON_OK) return r;
  const int n = static_cast<int>(in.size());
  std::vector<size_t> gb(n), pb(n);
  size_t total = 0;
  for (int k = 0; k < n; ++k) {
    const size_t numel = static_cast<size_t>(in[k].rows) * static_cast<size_t>(in[k].cols);
    gb[k] = numel * elem_bytes(in[k].gdt);
    pb[k] = numel * elem_bytes(in[k].pdt);
    total += gb[k];
  }
  std::vector<int> bnd;
  if (chunks <= 0) {
    bnd = ramp_bounds(gb);
  } else {
    chunks = std::min(chunks, n);
    bnd = chunk_bounds(gb, chunks);
  }
  const int nc = static_cast<int>(bnd.size()) - 1;
  std::vector<std::vector<MatIn>> sub(nc);
  size_t need = 0;
  for (int c = 0; c < nc; ++c) {
    sub[c].assign(in.begin() + bnd[c], in.begin() + bnd[c + 1]);
    need = std::max(need, make_layout(sub[c], o.steps, o.cc != 0.0f).bytes);
  }
  if (own_ws) {
    r = arena_get(dev, st, need, &ws);
    if (r != DMUON_OK) return r;
  } else {
    if (!ws) return fail(DMUON_ERR_INVALID_ARG, "NULL workspace");
    if (ws_bytes < need)
      return fail(DMUON_ERR_NO_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed",
                  ws_bytes, need);
    if (!aligned(ws, 256)) return fail(DMUON_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    r = check_device_ptr(dev, ws, 0, "the workspace", "argument");
    if (r != DMUON_OK) return r;
  }
  // Every group's plan before any copy is enqueued (a new plan's upload
  // writes library memory only).  The cache holds more plans than
  // DMUON_MAX_CHUNKS, so none of these is evicted by the others.
  std::vector<Plan*> plans(nc, nullptr);
  for (int c = 0; c < nc; ++c) {
    r = get_plan(sub[c], o.steps, o.cc != 0.0f, ws, dev, st, &plans[c]);
    if (r != DMUON_OK) return r;
  }
  CopyLanes* L = nullptr;
  r = copy_lanes(dev, &L);
  if (r != DMUON_OK) return r;

  cudaEvent_t start = L->ev[2 * DMUON_MAX_CHUNKS];
  cudaError_t e = cudaEventRecord(start, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(L->up, start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(L->down, start, 0);
  // All uploads back to back on one copy engine, one event per group.
  for (int c = 0; c < nc && e == cudaSuccess; ++c) {
    for (int k = bnd[c]; k < bnd[c + 1] && e == cudaSuccess; ++k)
      e = cudaMemcpyAsync(stage[k], hg[k], gb[k], cudaMemcpyHostToDevice, L->up);
    if (e == cudaSuccess) e = cudaEventRecord(L->ev[c], L->up);
  }
  if (e != cudaSuccess) return cuda_fail(e, "upload");
  for (int c = 0; c < nc; ++c) {
    e = cudaStreamWaitEvent(st, L->ev[c], 0);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
    r = prepare_plan(*plans[c], sub[c], st);
    if (r == DMUON_OK) r = launch_plan(*plans[c], o, st);
    if (r == DMUON_OK) r = finish_plan(*plans[c], st);
    if (r != DMUON_OK) return r;
    e = cudaEventRecord(L->ev[DMUON_MAX_CHUNKS + c], st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(L->down, L->ev[DMUON_MAX_CHUNKS + c], 0);
    for (int k = bnd[c]; k < bnd[c + 1] && e == cudaSuccess; ++k)
      if (hp[k]) e = cudaMemcpyAsync(hp[k], in[k].W, pb[k], cudaMemcpyDeviceToHost, L->down);
    if (e != cudaSuccess) return cuda_fail(e, "download");
  }
  // `stream` continues after the last download.
  e = cudaEventRecord(start, L->down);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, start, 0);
  if (e != cudaSuccess) return cuda_fail(e, "download completion");
  return DMUON_OK;
}

}  // namespace
}  // namespace dmuon

using namespace dmuon;

extern "C" {

int dmuon_muon_step_batched_ex(void* const params[], const void* const grads[], float* const bufs[],
                               const dmuon_shape shapes[], int count, float lr, float momentum,
                               int nesterov, float weight_decay, int ns_steps, void* workspace,
                               size_t ws_bytes, dmuon_stream_t stream) {
  t_last_error.clear();
  const StepOpts o = plain_opts(lr, momentum, nesterov, weight_decay, ns_steps);
  int r = check_opts(o);
  if (r != DMUON_OK) return r;
  std::vector<MatIn> in;
  r = gather(params, grads, bufs, shapes, count, ns_steps, DMUON_LR_PLAIN, &in);
  if (r != DMUON_OK) return r;
  return run(in, workspace, ws_bytes, false, o, reinterpret_cast<cudaStream_t>(stream));
}

int dmuon_muon_step_batched(void* const params[], const void* const grads[], float* const bufs[],
                            const dmuon_shape shapes[], int count, float lr, float momentum,
                            int nesterov, float weight_decay, int ns_steps, dmuon_stream_t stream) {
  t_last_error.clear();
  const StepOpts o = plain_opts(lr, momentum, nesterov, weight_decay, ns_steps);
  int r = check_opts(o);
  if (r != DMUON_OK) return r;
  std::vector<MatIn> in;
  r = gather(params, grads, bufs, shapes, count, ns_steps, DMUON_LR_PLAIN, &in);
  if (r != DMUON_OK) return r;
  return run(in, nullptr, 0, true, o, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace dmuon {
namespace {
// Options as the caller passed them.  The struct grew by ns_c at its end; a
// caller built against the earlier layout passes the shorter size and gets
// the cubic step.
constexpr size_t kOptsSizeNoQuintic = offsetof(dmuon_step_options, ns_c);

int read_opts(const dmuon_step_options* opts, StepOpts* o) {
  if (!opts) return fail(DMUON_ERR_INVALID_ARG, "NULL options");
  if (opts->struct_size != sizeof(dmuon_step_options) && opts->struct_size != kOptsSizeNoQuintic)
    return fail(DMUON_ERR_INVALID_ARG, "options.struct_size is %zu, this library expects %zu (use "
                "dmuon_step_options_default)", opts->struct_size, sizeof(dmuon_step_options));
  *o = plain_opts(opts->lr, opts->momentum, opts->nesterov, opts->weight_decay, opts->ns_steps);
  o->ca = opts->ns_a;
  o->cb = opts->ns_b;
  o->cc = opts->struct_size == sizeof(dmuon_step_options) ? opts->ns_c : 0.0f;
  o->lr_scale = opts->lr_scale;
  o->max_norm = opts->max_grad_norm;
  o->norm_out = opts->grad_norm_out;
  int r = check_opts(*o);
  if (r != DMUON_OK) return r;
  if (o->norm_out && !aligned(o->norm_out, 4)) return fail(DMUON_ERR_INVALID_ARG, "grad_norm_out misaligned");
  return DMUON_OK;
}
}  // namespace
}  // namespace dmuon

extern "C" {

void dmuon_step_options_default(dmuon_step_options* o) {
  if (!o) return;
  std::memset(o, 0, sizeof(*o));
  o->struct_size = sizeof(dmuon_step_options);
  o->lr = 0.02f;
  o->momentum = 0.95f;
  o->nesterov = 1;
  o->weight_decay = 0.0f;
  o->ns_steps = 5;
  o->ns_a = 1.5f;
  o->ns_b = -0.5f;
  o->lr_scale = DMUON_LR_PLAIN;
  o->max_grad_norm = 0.0f;
  o->grad_norm_out = nullptr;
  o->ns_c = 0.0f;
}

int dmuon_muon_step_batched_opts(void* const params[], const void* const grads[], float* const bufs[],
                                 const dmuon_shape shapes[], int count, const dmuon_step_options* opts,
                                 void* workspace, size_t ws_bytes, dmuon_stream_t stream) {
  t_last_error.clear();
  StepOpts o;
  int r = read_opts(opts, &o);
  if (r != DMUON_OK) return r;
  std::vector<MatIn> in;
  r = gather(params, grads, bufs, shapes, count, opts->ns_steps, o.lr_scale, &in);
  if (r != DMUON_OK) return r;
  return run(in, workspace, ws_bytes, workspace == nullptr, o, reinterpret_cast<cudaStream_t>(stream));
}

int dmuon_muon_step_batched_reduce(void* const params[], const void* const grads[], float* const bufs[],
                                   const dmuon_shape shapes[], int count, int world,
                                   const dmuon_step_options* opts, void* workspace, size_t ws_bytes,
                                   dmuon_stream_t stream) {
  t_last_error.clear();
  StepOpts o;
  int r = read_opts(opts, &o);
  if (r != DMUON_OK) return r;
  if (world < 1 || world > 64) return fail(DMUON_ERR_INVALID_ARG, "world must be in [1, 64]");
  if (count > 0 && !grads) return fail(DMUON_ERR_INVALID_ARG, "NULL array argument");
  // Rank 0's pointers stand for the gradients in the argument checks.
  std::vector<MatIn> in;
  r = gather(params, grads, bufs, shapes, count, opts->ns_steps, o.lr_scale, &in);
  if (r != DMUON_OK) return r;
  size_t k = 0;
  for (int i = 0; i < count; ++i) {
    const bool has = grads[i] != nullptr;
    const size_t eb = (shapes[i].grad_dtype == DMUON_BF16) ? 2 : 4;
    for (int q = 1; q < world; ++q) {
      const void* g = grads[static_cast<int64_t>(q) * count + i];
      if ((g != nullptr) != has)
        return fail(DMUON_ERR_INVALID_ARG, "matrix %d: rank %d's gradient is %s while rank 0's is %s", i, q,
                    g ? "given" : "NULL", has ? "given" : "NULL");
      if (g && !aligned(g, eb))
        return fail(DMUON_ERR_INVALID_ARG, "matrix %d: rank %d's gradient is misaligned", i, q);
    }
    if (!has) continue;
    if (world > 1)
      for (int q = 0; q < world; ++q) in[k].gr.push_back(grads[static_cast<int64_t>(q) * count + i]);
    ++k;
  }
  return run(in, workspace, ws_bytes, workspace == nullptr, o, reinterpret_cast<cudaStream_t>(stream));
}

int dmuon_muon_step_batched_host(void* const params[], void* const grads[], float* const bufs[],
                                 const void* const host_grads[], void* const host_params[],
                                 const dmuon_shape shapes[], int count, const dmuon_step_options* opts,
                                 int chunks, void* workspace, size_t ws_bytes, dmuon_stream_t stream) {
  t_last_error.clear();
  StepOpts o;
  int r = read_opts(opts, &o);
  if (r != DMUON_OK) return r;
  if (o.max_norm != 0.0f)
    return fail(DMUON_ERR_UNSUPPORTED, "gradient clipping needs every gradient before the first "
                "update; use dmuon_muon_step_batched_opts");
  if (chunks > DMUON_MAX_CHUNKS)
    return fail(DMUON_ERR_INVALID_ARG, "chunks must be <= %d", DMUON_MAX_CHUNKS);
  if (count > 0 && (!host_grads || !host_params || !grads))
    return fail(DMUON_ERR_INVALID_ARG, "NULL array argument");
  std::vector<MatIn> in;
  // Checked as given, then the device staging buffers stand for the
  // gradients in the update.
  r = gather(params, host_grads, bufs, shapes, count, opts->ns_steps, o.lr_scale, &in);
  if (r != DMUON_OK) return r;
  std::vector<const void*> hg;
  std::vector<void*> hp, stage;
  for (int i = 0; i < count; ++i) {
    if (!host_grads[i]) continue;
    if (!grads[i]) return fail(DMUON_ERR_INVALID_ARG, "matrix %d: NULL device gradient buffer", i);
    if (!page_locked(host_grads[i]))
      return fail(DMUON_ERR_UNSUPPORTED, "matrix %d: host gradient is not page-locked memory", i);
    if (host_params[i] && !page_locked(host_params[i]))
      return fail(DMUON_ERR_UNSUPPORTED, "matrix %d: host parameter buffer is not page-locked memory", i);
    const size_t eb = elem_bytes(shapes[i].grad_dtype);
    if (!aligned(grads[i], eb))
      return fail(DMUON_ERR_INVALID_ARG, "matrix %d: device gradient buffer misaligned", i);
    MatIn& x = in[hg.size()];
    x.G = grads[i];
    hg.push_back(host_grads[i]);
    hp.push_back(host_params[i]);
    stage.push_back(grads[i]);
  }
  return run_host(in, hg, hp, stage, chunks, workspace, ws_bytes, workspace == nullptr, o,
                  reinterpret_cast<cudaStream_t>(stream));
}

size_t dmuon_workspace_bytes(const dmuon_shape shapes[], int count, int ns_steps) {
  if (count <= 0 || !shapes || ns_steps < 0 || ns_steps > DMUON_MAX_STEPS) return 0;
  std::vector<MatIn> in(count);
  for (int i = 0; i < count; ++i) {
    MatIn& x = in[i];
    x.W = x.buf = nullptr;
    x.G = nullptr;
    x.rows = shapes[i].rows;
    x.cols = shapes[i].cols;
    x.pdt = shapes[i].param_dtype;
    x.gdt = shapes[i].grad_dtype;
    x.mode = kModeMuon;
    if (x.rows < 1 || x.cols < 1 || (x.pdt != DMUON_BF16 && x.pdt != DMUON_F32)) return 0;
  }
  return make_layout(in, ns_steps).bytes;
}

size_t dmuon_workspace_bytes_opts(const dmuon_shape shapes[], int count, const dmuon_step_options* opts) {
  if (!opts || (opts->struct_size != sizeof(dmuon_step_options) && opts->struct_size != kOptsSizeNoQuintic))
    return 0;
  const int steps = opts->ns_steps;
  if (count <= 0 || !shapes || steps < 0 || steps > DMUON_MAX_STEPS) return 0;
  const bool quintic = opts->struct_size == sizeof(dmuon_step_options) && opts->ns_c != 0.0f;
  std::vector<MatIn> in(count);
  for (int i = 0; i < count; ++i) {
    MatIn& x = in[i];
    x.rows = shapes[i].rows;
    x.cols = shapes[i].cols;
    x.pdt = shapes[i].param_dtype;
    x.gdt = shapes[i].grad_dtype;
    x.mode = kModeMuon;
    if (x.rows < 1 || x.cols < 1 || (x.pdt != DMUON_BF16 && x.pdt != DMUON_F32)) return 0;
  }
  return make_layout(in, steps, quintic).bytes;
}

static int ortho_input(void* X, int64_t m, int64_t n, int steps, int dtype, std::vector<MatIn>* in) {
  if (steps < 0 || steps > DMUON_MAX_STEPS)
    return fail(DMUON_ERR_INVALID_ARG, "steps must be in [0, %d]", DMUON_MAX_STEPS);
  MatIn x;
  x.W = X;
  x.G = X;
  x.buf = nullptr;
  x.rows = m;
  x.cols = n;
  x.pdt = dtype;
  x.gdt = dtype;
  x.mode = kModeOrtho;
  const int r = check_matrix(x, 0);
  if (r != DMUON_OK) return r;
  in->push_back(x);
  return DMUON_OK;
}

int dmuon_ns_orthogonalize_ex(void* X, int64_t m, int64_t n, int steps, int dtype, void* workspace,
                              size_t ws_bytes, dmuon_stream_t stream) {
  t_last_error.clear();
  std::vector<MatIn> in;
  int r = ortho_input(X, m, n, steps, dtype, &in);
  if (r != DMUON_OK) return r;
  return run(in, workspace, ws_bytes, false, plain_opts(0.0f, 0.0f, 0, 0.0f, steps),
             reinterpret_cast<cudaStream_t>(stream));
}

int dmuon_ns_orthogonalize(void* X, int64_t m, int64_t n, int steps, dmuon_stream_t stream) {
  t_last_error.clear();
  std::vector<MatIn> in;
  int r = ortho_input(X, m, n, steps, DMUON_BF16, &in);
  if (r != DMUON_OK) return r;
  return run(in, nullptr, 0, true, plain_opts(0.0f, 0.0f, 0, 0.0f, steps),
             reinterpret_cast<cudaStream_t>(stream));
}

size_t dmuon_ns_workspace_bytes(int64_t m, int64_t n, int dtype) {
  if (m < 1 || n < 1 || (dtype != DMUON_BF16 && dtype != DMUON_F32)) return 0;
  std::vector<MatIn> in(1);
  in[0].rows = m;
  in[0].cols = n;
  in[0].pdt = in[0].gdt = dtype;
  in[0].mode = kModeOrtho;
  return make_layout(in, 2).bytes;
}

const char* dmuon_last_error(void) { return t_last_error.c_str(); }

const char* dmuon_backend_string(void) {
  return "cubic Newton-Schulz · tcgen05 UMMA SYRK (upper 256x256 tiles, two halves sharing B) + GEMM "
         "128x256 (fused combine/update, transposed lower A) · TMA 128B-swizzle · TMEM · sm_100a";
}

int dmuon_device_status(int clear) {
  t_last_error.clear();
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (clear) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
  }
  return v;
}

void dmuon_release_cache(void) {
  std::lock_guard<std::mutex> lk(g_api_mu);
  cudaDeviceSynchronize();
  g_plans.clear();
  for (auto& kv : g_arenas)
    if (kv.second.ptr) cudaFree(kv.second.ptr);
  g_arenas.clear();
  for (void* p : g_parked) cudaFree(p);
  g_parked.clear();
  for (DeviceInfo& d : g_dev)
    if (d.pool) cudaMemPoolTrimTo(d.pool, 0);
}

int64_t dmuon_plan_builds(void) {
  std::lock_guard<std::mutex> lk(g_api_mu);
  return g_plan_builds;
}

int dmuon_debug_last_plan(int* kernels, int max_groups) {
  std::lock_guard<std::mutex> lk(g_api_mu);
  if (g_plans.empty()) return 0;
  const Plan& P = *g_plans.front();
  const int n = static_cast<int>(P.groups.size());
  for (int i = 0; i < n && i < max_groups; ++i)
    if (kernels)
      kernels[i] = (P.groups[i].syrk256 ? DMUON_PLAN_SYRK256 : 0) | (P.groups[i].gemm_pair ? DMUON_PLAN_GEMM_PAIR : 0) |
                   (P.quintic && P.groups[i].square256 ? DMUON_PLAN_SQUARE256 : 0);
  return n;
}

int dmuon_debug_check_pointer(const void* p) {
  t_last_error.clear();
  if (p == nullptr) return fail(DMUON_ERR_INVALID_ARG, "NULL pointer");
  const int r = classify_pointer(p);
  if (r != DMUON_OK) return fail(r, "not device memory");
  return DMUON_OK;
}

int dmuon_adamw_step_batched(void* const params[], const void* const grads[], float* const exp_avgs[],
                             float* const exp_avg_sqs[], const dmuon_tensor_desc descs[], int count,
                             float lr, float beta1, float beta2, float eps, float weight_decay,
                             int64_t step, dmuon_stream_t stream) {
  t_last_error.clear();
  if (count < 0) return fail(DMUON_ERR_INVALID_ARG, "count must be >= 0");
  if (count == 0) return DMUON_OK;
  if (!params || !grads || !exp_avgs || !exp_avg_sqs || !descs)
    return fail(DMUON_ERR_INVALID_ARG, "NULL array argument");
  if (!std::isfinite(lr) || !std::isfinite(weight_decay) || !(beta1 >= 0.0f && beta1 < 1.0f) ||
      !(beta2 >= 0.0f && beta2 < 1.0f) || !(eps > 0.0f) || !std::isfinite(eps))
    return fail(DMUON_ERR_INVALID_ARG, "need finite lr and weight_decay, betas in [0, 1), eps > 0");
  if (step < 1) return fail(DMUON_ERR_INVALID_ARG, "step must be >= 1");
  std::vector<AdamTensor> ts;
  ts.reserve(count);
  for (int i = 0; i < count; ++i) {
    if (grads[i] == nullptr) continue;
    const dmuon_tensor_desc& d = descs[i];
    if (d.numel < 1) return fail(DMUON_ERR_INVALID_ARG, "tensor %d: numel must be >= 1", i);
    if ((d.param_dtype != DMUON_BF16 && d.param_dtype != DMUON_F32) ||
        (d.grad_dtype != DMUON_BF16 && d.grad_dtype != DMUON_F32))
      return fail(DMUON_ERR_UNSUPPORTED, "tensor %d: dtype must be DMUON_BF16 or DMUON_F32", i);
    if (!params[i] || !exp_avgs[i] || !exp_avg_sqs[i])
      return fail(DMUON_ERR_INVALID_ARG, "tensor %d: NULL pointer", i);
    if (!aligned(params[i], elem_bytes(d.param_dtype)) || !aligned(grads[i], elem_bytes(d.grad_dtype)) ||
        !aligned(exp_avgs[i], 4) || !aligned(exp_avg_sqs[i], 4))
      return fail(DMUON_ERR_INVALID_ARG, "tensor %d: pointer not aligned to its element size", i);
    AdamTensor t;
    t.p = params[i];
    t.g = grads[i];
    t.m = exp_avgs[i];
    t.v = exp_avg_sqs[i];
    t.numel = d.numel;
    t.item0 = 0;
    t.p_bf16 = d.param_dtype == DMUON_BF16;
    t.g_bf16 = d.grad_dtype == DMUON_BF16;
    ts.push_back(t);
  }
  if (ts.empty()) return DMUON_OK;
  std::lock_guard<std::mutex> lk(g_api_mu);
  int dev = 0;
  int r = current_device(&dev);
  if (r != DMUON_OK) return r;
  for (size_t k = 0; k < ts.size() && r == DMUON_OK; ++k) {
    const int i = static_cast<int>(k);
    r = check_device_ptr(dev, ts[k].p, i, "the parameter", "tensor");
    if (r == DMUON_OK) r = check_device_ptr(dev, ts[k].g, i, "the gradient", "tensor");
    if (r == DMUON_OK) r = check_device_ptr(dev, ts[k].m, i, "exp_avg", "tensor");
    if (r == DMUON_OK) r = check_device_ptr(dev, ts[k].v, i, "exp_avg_sq", "tensor");
  }
  if (r != DMUON_OK) return r;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const double bc1 = 1.0 - std::pow(static_cast<double>(beta1), static_cast<double>(step));
  const double bc2 = 1.0 - std::pow(static_cast<double>(beta2), static_cast<double>(step));
  std::unique_ptr<AdamParams> ap(new AdamParams());
  ap->b1 = beta1;
  ap->b2 = beta2;
  ap->c1 = 1.0f - beta1;
  ap->c2 = 1.0f - beta2;
  ap->eps = eps;
  ap->decay = 1.0f - lr * weight_decay;
  ap->step_size = static_cast<float>(static_cast<double>(lr) / bc1);
  ap->inv_bc2_sqrt = static_cast<float>(1.0 / std::sqrt(bc2));
  for (size_t first = 0; first < ts.size(); first += kAdamMaxTensors) {
    const int n = static_cast<int>(std::min<size_t>(kAdamMaxTensors, ts.size() - first));
    int64_t items = 0;
    for (int k = 0; k < n; ++k) {
      ap->t[k] = ts[first + k];
      ap->t[k].item0 = items;
      items += cdiv(ap->t[k].numel, kAdamChunk);
    }
    ap->count = n;
    ap->nitems = items;
    const int grid = static_cast<int>(std::min<int64_t>(items, static_cast<int64_t>(g_dev[dev].sms) * 8));
    LaunchScope ls(st, DMUON_KERNEL_ADAMW);
    adamw_kernel<<<grid, kPThreads, 0, st>>>(*ap);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return DMUON_OK;
}

static int clip_check(const dmuon_grad_desc descs[], int count, int nseg) {
  if (count < 0) return fail(DMUON_ERR_INVALID_ARG, "count must be >= 0");
  if (nseg < 1 || nseg > DMUON_MAX_SEGMENTS)
    return fail(DMUON_ERR_INVALID_ARG, "nseg must be in [1, %d]", DMUON_MAX_SEGMENTS);
  if (count > 0 && !descs) return fail(DMUON_ERR_INVALID_ARG, "NULL array argument");
  for (int i = 0; i < count; ++i) {
    const dmuon_grad_desc& d = descs[i];
    if (d.numel < 1) return fail(DMUON_ERR_INVALID_ARG, "tensor %d: numel must be >= 1", i);
    if (d.dtype != DMUON_BF16 && d.dtype != DMUON_F32)
      return fail(DMUON_ERR_UNSUPPORTED, "tensor %d: dtype must be DMUON_BF16 or DMUON_F32", i);
    if (d.segment < 0 || d.segment >= nseg)
      return fail(DMUON_ERR_INVALID_ARG, "tensor %d: segment %d is outside [0, %d)", i, d.segment, nseg);
  }
  return DMUON_OK;
}

// Scratch of one clip call: one fp64 partial per 32 KB work item, then the
// per-segment coefficients.
static int64_t clip_items_of(const dmuon_grad_desc& d) {
  return cdiv(d.numel * elem_bytes(d.dtype), kClipItemBytes);
}
static size_t clip_scratch_bytes(const dmuon_grad_desc descs[], int count, int nseg, size_t* coef_off) {
  int64_t items = 0;
  for (int i = 0; i < count; ++i) items += clip_items_of(descs[i]);
  const size_t off = align_up(sizeof(double) * static_cast<size_t>(std::max<int64_t>(items, 1)), 256);
  if (coef_off) *coef_off = off;
  return off + align_up(sizeof(float) * nseg, 256);
}

size_t dmuon_clip_workspace_bytes(const dmuon_grad_desc descs[], int count, int nseg) {
  if (clip_check(descs, count, nseg) != DMUON_OK) return 0;
  return clip_scratch_bytes(descs, count, nseg, nullptr);
}

int dmuon_clip_grad_norm_buckets(void* const grads[], const dmuon_grad_desc descs[], int count,
                                 const float max_norms[], int nseg, float* norms_out, float* coefs_out,
                                 void* workspace, size_t ws_bytes, dmuon_stream_t stream) {
  t_last_error.clear();
  int r = clip_check(descs, count, nseg);
  if (r != DMUON_OK) return r;
  if (count > 0 && !grads) return fail(DMUON_ERR_INVALID_ARG, "NULL array argument");
  if (!max_norms) return fail(DMUON_ERR_INVALID_ARG, "NULL max_norms");
  for (int s = 0; s < nseg; ++s)
    if (!(max_norms[s] > 0.0f))
      return fail(DMUON_ERR_INVALID_ARG, "max_norms[%d] must be > 0 (+inf measures without clipping)", s);
  if ((norms_out && !aligned(norms_out, 4)) || (coefs_out && !aligned(coefs_out, 4)))
    return fail(DMUON_ERR_INVALID_ARG, "norms_out / coefs_out misaligned");
  // Tensors with a gradient, sorted by segment (stable): each segment's work
  // items form one contiguous range.
  std::vector<int> idx;
  for (int i = 0; i < count; ++i) {
    if (!grads[i]) continue;
    if (!aligned(grads[i], elem_bytes(descs[i].dtype)))
      return fail(DMUON_ERR_INVALID_ARG, "tensor %d: pointer not aligned to its element size", i);
    idx.push_back(i);
  }
  std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) { return descs[a].segment < descs[b].segment; });
  std::vector<ClipTensor> ts(idx.size());
  std::unique_ptr<ClipFinalizeParams> fp(new ClipFinalizeParams());
  int64_t items = 0;
  int seg = 0;
  fp->seg_item0[0] = 0;
  for (size_t k = 0; k < idx.size(); ++k) {
    const dmuon_grad_desc& d = descs[idx[k]];
    while (seg < d.segment) fp->seg_item0[++seg] = items;
    ts[k].g = grads[idx[k]];
    ts[k].numel = d.numel;
    ts[k].item0 = items;
    ts[k].seg = d.segment;
    ts[k].bf16 = d.dtype == DMUON_BF16;
    items += clip_items_of(d);
  }
  while (seg < nseg) fp->seg_item0[++seg] = items;
  for (int s = 0; s < nseg; ++s) fp->max_norm[s] = max_norms[s];
  size_t coef_off = 0;
  const size_t need = clip_scratch_bytes(descs, count, nseg, &coef_off);

  std::lock_guard<std::mutex> lk(g_api_mu);
  int dev = 0;
  r = current_device(&dev);
  if (r != DMUON_OK) return r;
  for (size_t k = 0; k < ts.size() && r == DMUON_OK; ++k)
    r = check_device_ptr(dev, ts[k].g, idx[k], "the gradient", "tensor");
  if (r == DMUON_OK) r = check_device_ptr(dev, norms_out, 0, "norms_out", "output");
  if (r == DMUON_OK) r = check_device_ptr(dev, coefs_out, 0, "coefs_out", "output");
  if (r == DMUON_OK) r = check_device_ptr(dev, workspace, 0, "the workspace", "argument");
  if (r != DMUON_OK) return r;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void* ws = workspace;
  if (!ws) {
    r = arena_get(dev, st, need, &ws);
    if (r != DMUON_OK) return r;
  } else {
    if (ws_bytes < need)
      return fail(DMUON_ERR_NO_WORKSPACE, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes, need);
    if (!aligned(ws, 256)) return fail(DMUON_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  }
  double* partials = static_cast<double*>(ws);
  float* coef = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + coef_off);
  fp->partials = partials;
  fp->coef = coef;
  fp->norms_out = norms_out;
  fp->coefs_out = coefs_out;
  const int sms = g_dev[dev].sms;
  std::unique_ptr<ClipBucketParams> cp(new ClipBucketParams());
  cp->partials = partials;
  cp->coef = coef;
  // The tensors in launches of at most kClipMaxTensors, for the norm pass and
  // then (after the coefficients) for the scale pass.
  auto launch_all = [&](bool scale) {
    for (size_t first = 0; first < ts.size(); first += kClipMaxTensors) {
      const int n = static_cast<int>(std::min<size_t>(kClipMaxTensors, ts.size() - first));
      for (int k = 0; k < n; ++k) cp->t[k] = ts[first + k];
      cp->count = n;
      cp->item_begin = ts[first].item0;
      cp->item_end = (first + n < ts.size()) ? ts[first + n].item0 : items;
      const int64_t ni = cp->item_end - cp->item_begin;
      if (ni <= 0) continue;
      // four resident blocks per SM (64 registers a thread): one wave of them
      const int grid = static_cast<int>(std::min<int64_t>(ni, static_cast<int64_t>(sms) * 4));
      LaunchScope ls(st, DMUON_KERNEL_CLIP);
      if (scale) clip_scale_kernel<<<grid, kPThreads, 0, st>>>(*cp);
      else clip_norm_kernel<<<grid, kPThreads, 0, st>>>(*cp);
    }
  };
  launch_all(false);
  {
    LaunchScope ls(st, DMUON_KERNEL_CLIP);
    clip_finalize_kernel<<<nseg, kClipFinThreads, 0, st>>>(*fp);
  }
  launch_all(true);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return DMUON_OK;
}

int dmuon_stage_timing(int enable) {
  std::lock_guard<std::mutex> lk(g_api_mu);
  g_timing = enable != 0;
  return DMUON_OK;
}

int dmuon_stage_times(double* ms, int64_t* launches, int n, int reset) {
  t_last_error.clear();
  std::lock_guard<std::mutex> lk(g_api_mu);
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  for (const Bracket& br : g_brackets) {
    float t = 0.0f;
    if (cudaEventElapsedTime(&t, br.a, br.b) == cudaSuccess) {
      g_kind_ms[br.kind] += t;
      g_kind_n[br.kind] += 1;
    }
    if (br.own_a) g_event_pool.push_back(br.a);
    g_event_pool.push_back(br.b);
  }
  g_brackets.clear();
  for (int k = 0; k < n && k < DMUON_KERNEL_KINDS; ++k) {
    if (ms) ms[k] = g_kind_ms[k];
    if (launches) launches[k] = g_kind_n[k];
  }
  if (reset)
    for (int k = 0; k < DMUON_KERNEL_KINDS; ++k) { g_kind_ms[k] = 0.0; g_kind_n[k] = 0; }
  return DMUON_OK;
}

int64_t dmuon_launch_count(void) {
  std::lock_guard<std::mutex> lk(g_api_mu);
  return g_launches;
}

void dmuon_debug_fail_allocations(int n) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_fail_allocs = n > 0 ? n : 0;
}

int dmuon_debug_partition(const dmuon_shape shapes[], int count, int which, int* bounds, int cap) {
  t_last_error.clear();
  if (!shapes || !bounds || count < 1 || cap < 2 || (which != 0 && which != 1))
    return fail(DMUON_ERR_INVALID_ARG, "bad arguments");
  std::vector<MatIn> in(count);
  std::vector<size_t> gb(count);
  for (int i = 0; i < count; ++i) {
    in[i].rows = shapes[i].rows;
    in[i].cols = shapes[i].cols;
    in[i].pdt = shapes[i].param_dtype;
    in[i].gdt = shapes[i].grad_dtype;
    if (in[i].rows < 1 || in[i].cols < 1 || (in[i].gdt != DMUON_BF16 && in[i].gdt != DMUON_F32))
      return fail(DMUON_ERR_INVALID_ARG, "bad shape %d", i);
    gb[i] = static_cast<size_t>(in[i].rows) * static_cast<size_t>(in[i].cols) * elem_bytes(in[i].gdt);
  }
  const std::vector<int> bnd = which == 0 ? step_groups(in, false) : ramp_bounds(gb);
  if (static_cast<int>(bnd.size()) > cap) return fail(DMUON_ERR_INVALID_ARG, "cap too small");
  for (size_t k = 0; k < bnd.size(); ++k) bounds[k] = bnd[k];
  return static_cast<int>(bnd.size()) - 1;
}

int dmuon_debug_wait_timeout(int limit_us, dmuon_stream_t stream) {
  t_last_error.clear();
  if (limit_us < 1 || limit_us > 10000000)
    return fail(DMUON_ERR_INVALID_ARG, "limit_us must be in [1, 1e7]");
  std::lock_guard<std::mutex> lk(g_api_mu);
  int dev = 0;
  int r = current_device(&dev);
  if (r != DMUON_OK) return r;
  ++g_launches;
  wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      g_dev[dev].err, static_cast<uint64_t>(limit_us) * 1000ull);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return DMUON_OK;
}

}  // extern "C"

// ======================================================================
// Allocation-free orthogonalisation.
//
// Some callers may not allocate device memory at all: code that runs inside
// a host framework which has already reserved all device memory for its own
// pool, plugins whose sandbox forbids cudaMalloc, and latency-critical paths
// where cudaMalloc/cudaFree may block on, or synchronise with, the device.
// For them dmuon_ns_orthogonalize_noalloc() takes its scratch (iterates,
// Gram matrix, norm partials and the small launch description) from the
// fixed array below, which the CUDA module reserves on every device that
// loads this library and keeps until the process exits.
// ======================================================================
namespace dmuon {

constexpr size_t kStaticScratchBytes = 32ull << 20;   // 32 MiB in total
constexpr size_t kStaticPlanBytes = 16384;            // launch description at the front

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {

// Device address of g_static_scratch, fetched once per device.  The host-side
// name of a __device__ array is only a stand-in for it, so kernels must be
// given this address instead.
uint8_t* g_static_addr[64] = {nullptr};

int static_scratch_address(int dev, uint8_t** out) {
  if (g_static_addr[dev] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    g_static_addr[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_static_addr[dev];
  return DMUON_OK;
}

// Launch description of one matrix, laid out as the device reads it.
struct alignas(128) StaticPlan {
  MatDesc desc;
  int order[2];
  int syrk_prefix[2];
  int gemm_prefix[2];
  int pad_[2];
  int64_t pprefix[2];
  alignas(64) MatMaps maps;
};
static_assert(sizeof(StaticPlan) <= kStaticPlanBytes, "launch description does not fit");

}  // namespace
}  // namespace dmuon

extern "C" int dmuon_ns_orthogonalize_noalloc(void* X, int64_t m, int64_t n, int steps,
                                              dmuon_stream_t stream) {
  using namespace dmuon;
  t_last_error.clear();
  std::vector<MatIn> in;
  int r = ortho_input(X, m, n, steps, DMUON_BF16, &in);
  if (r != DMUON_OK) return r;
  const Layout L = make_layout(in, steps);
  const size_t room = kStaticScratchBytes - kStaticPlanBytes;
  if (L.bytes > room)
    return fail(DMUON_ERR_UNSUPPORTED,
                "dmuon_ns_orthogonalize_noalloc: a %lld x %lld matrix with %d steps needs %zu "
                "bytes of scratch; the static scratch holds %zu (use dmuon_ns_orthogonalize_ex)",
                (long long)m, (long long)n, steps, L.bytes, room);
  std::lock_guard<std::mutex> lk(g_api_mu);
  int dev = 0;
  r = current_device(&dev);
  if (r != DMUON_OK) return r;
  r = check_device_ptr(dev, X, 0, "X");
  if (r != DMUON_OK) return r;
  uint8_t* base = nullptr;
  r = static_scratch_address(dev, &base);
  if (r != DMUON_OK) return r;
  uint8_t* ws = base + kStaticPlanBytes;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  // Host image of the launch description.
  const MatLayout& ml = L.mats[0];
  const GroupLayout& g = L.groups[0];
  StaticPlan sp;
  std::memset(&sp, 0, sizeof(sp));
  MatDesc& d = sp.desc;
  d.W = X; d.G = X; d.buf = nullptr;
  d.rows = m; d.cols = n;
  d.ldx = ml.ldx; d.lda = ml.lda;
  d.X[0] = ws + ml.x0;
  d.X[1] = (ml.x1 != SIZE_MAX) ? ws + ml.x1 : nullptr;
  d.Xop[0] = d.X[0];
  d.Xop[1] = d.X[1];
  d.A = (ml.a != SIZE_MAX) ? ws + ml.a : nullptr;
  d.scale = reinterpret_cast<float*>(ws + g.scales);
  d.lr_mult = 1.0f;
  d.m = static_cast<int>(ml.m); d.n = static_cast<int>(ml.n);
  d.T = m > n ? 1 : 0;
  d.mode = kModeOrtho;
  d.g_bf16 = 1;
  d.vec4 = (n % 4 == 0) && aligned(X, 16);
  d.ptiles_c = static_cast<int>(ml.ptiles_c);
  const bool big_syrk = use_syrk256(syrk_tiles_of(ml.m), syrk256_tiles_of(ml.m), g_dev[dev].sms);
  const int syrk_tiles = static_cast<int>(big_syrk ? syrk256_tiles_of(ml.m) : syrk_tiles_of(ml.m));
  const int gemm_tiles = static_cast<int>(gemm_tiles_of(ml.m, ml.n));
  sp.order[0] = 0;
  sp.syrk_prefix[1] = syrk_tiles;
  sp.gemm_prefix[1] = gemm_tiles;
  sp.pprefix[1] = ml.ptiles;
  const int BK = 64;   // bf16: 128-byte K slices
  bool okm = true;
  // As in the regular plans: the GEMM's B operand in one 3-D load when n % 64 == 0.
  d.b3d = (ml.n % 64 == 0) ? 1 : 0;
  for (int b = 0; b < 2 && d.b3d; ++b)
    if (d.X[b] && !encode_mn3d(&sp.maps.xmn[b], d.X[b], ml.n, ml.m, ml.ldx)) d.b3d = 0;
  for (int b = 0; b < 2; ++b) {
    void* xb = d.X[b];
    if (!xb) {
      sp.maps.xk[b] = sp.maps.xk[0]; sp.maps.xkw[b] = sp.maps.xkw[0]; sp.maps.xmn[b] = sp.maps.xmn[0];
      continue;
    }
    okm &= encode_2d(&sp.maps.xk[b], DMUON_BF16, xb, ml.n, ml.m, ml.ldx, BK, kBM);
    okm &= encode_2d(&sp.maps.xkw[b], DMUON_BF16, xb, ml.n, ml.m, ml.ldx, BK, kBN);
    if (!d.b3d) okm &= encode_2d(&sp.maps.xmn[b], DMUON_BF16, xb, ml.n, ml.m, ml.ldx, BK, BK);
  }
  if (d.A) {
    okm &= encode_2d(&sp.maps.a, DMUON_BF16, d.A, ml.m, ml.m, ml.lda, BK, kBM);
    okm &= encode_2d(&sp.maps.amn, DMUON_BF16, d.A, ml.m, ml.m, ml.lda, BK, BK);
  }
  if (!okm) return fail(DMUON_ERR_CUDA, "cuTensorMapEncodeTiled failed");

  // The launch description travels as kernel parameters of an upload kernel
  // on the caller's stream: ordered after any earlier call on it, no host
  // staging memory.  The stage kernels acquire the tensor maps before use.
  enqueue_upload(base, reinterpret_cast<const uint8_t*>(&sp), sizeof(sp), st);
  const StaticPlan* dsp = reinterpret_cast<const StaticPlan*>(base);

  const DeviceInfo& di = g_dev[dev];
  ElemParams ep;
  ep.mats = &dsp->desc;
  ep.ptile_prefix = dsp->pprefix;
  ep.partials = reinterpret_cast<float*>(ws + g.partials);
  ep.nmat = 1;
  ep.ntiles = ml.ptiles;
  ep.mu = 0.0f;
  ep.nesterov = 0;
  ep.lr = 0.0f;
  ep.wd = 0.0f;
  ep.clip = nullptr;
  ep.gpartials = nullptr;
  const int pgrid = static_cast<int>(std::min<int64_t>(ml.ptiles, static_cast<int64_t>(di.sms) * 8));
  prologue_kernel<__nv_bfloat16><<<pgrid, kPThreads, kProSmemBytes, st>>>(ep);
  finalize_kernel<<<1, 32, 0, st>>>(ep);
  g_launches += 2;
  if (steps == 0) {
    apply_kernel<__nv_bfloat16><<<pgrid, kPThreads, 0, st>>>(ep);
    ++g_launches;
  } else {
    NsParams np;
    np.mats = &dsp->desc;
    np.maps = &dsp->maps;
    np.order = dsp->order;
    np.nmat = 1;
    np.lr = 0.0f;
    np.wd = 0.0f;
    np.ca = 1.5f;
    np.cb = -0.5f;
    np.cc = 0.0f;
    np.quintic = 0;
    np.mirror = 0;
    np.a_upper = 1;
    np.diag_full = 0;
    np.err = di.err;
    np.wait_limit_ns = kWaitLimitNs;
    for (int s = 0; s < steps; ++s) {
      np.cur = s & 1;
      np.first = s == 0;
      np.last = s == steps - 1;
      np.tile_prefix = dsp->syrk_prefix;
      np.ntiles = syrk_tiles;
      if (big_syrk)
        syrk256_kernel<__nv_bfloat16><<<std::min(np.ntiles, di.sms), kNsThreads, kS2SmemBytes, st>>>(np);
      else
        launch_ns_stage<kSyrk, __nv_bfloat16>(np, di, st);
      np.tile_prefix = dsp->gemm_prefix;
      np.ntiles = gemm_tiles;
      launch_ns_stage<kGemm, __nv_bfloat16>(np, di, st);
      g_launches += 2;
    }
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
  return DMUON_OK;
}
