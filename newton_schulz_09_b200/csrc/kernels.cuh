// Kernels of the batched Muon update on sm_100a.
//
//   prologue_kernel     momentum, Nesterov input, per-tile sum of squares and
//                       the (transposed when rows > cols) copy of M into the
//                       iteration's X buffer.                     [HBM bound]
//   finalize_kernel     fixed-order sum of the tile partials per matrix and
//                       s = 1 / (||M||_F + 1e-7).
//   ns_stage_kernel     one Newton-Schulz stage for every matrix of a group
//                       in one persistent launch:
//                         SYRK  A = s^2 X X^T  (upper tiles; mirrored only for
//                               quintic groups that do not run on CTA pairs)
//                         SQUARE P = b A + c A A  (quintic coefficients only)
//                         GEMM  X' = c (1.5 X - 0.5 A X), or on the last step
//                               the weight update / output write.   [tensor]
//   apply_kernel        the update for ns_steps == 0 (X = s M).
//   grad_norm_kernel,   Muon-only global-norm gradient clipping: per-item
//   clip_coef_kernel    sums of g^2 (fp64), then the clip coefficient.
//   adamw_kernel        AdamW of the parameters Muon does not orthogonalise.
//   clip_*_kernel       per-segment gradient clipping (norms, coefficients,
//                       in-place scaling) of several gradient groups.
//   wait_timeout_kernel test kernel of the bounded-wait path.
//
// Sources: DMuon blog post "DMuon：让矩阵正交化优化器达到接近 AdamW 的分布式训练开销",
// sections "Muon 核心：Newton-Schulz 迭代" (normalisation, cubic step,
// transpose rule) and "代码实现 / Vanilla Muon" (momentum, update); DMuon
// training guide "训练指南", section "超参数指南" (Nesterov input).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace dmuon {

// ------------------------------------------------------------------ layout
constexpr int kBM = 128;           // tile rows (UMMA M, TMEM lanes)
constexpr int kBN = 256;           // tile cols (UMMA N, TMEM columns per accumulator)
constexpr int kStages = 4;         // smem pipeline depth
constexpr int kAStageBytes = kBM * 128;   // one 128-byte K slice of 128 rows
constexpr int kBStageBytes = kBN * 128;   // one 128-byte K slice of 256 rows
constexpr int kTmemCols = 2 * kBN;        // double-buffered fp32 accumulator
constexpr int kNsThreads = 192;           // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kEpiSlotBytes = kBM * 128;  // one 128-row x 128-byte output quarter (bf16 GEMM)
constexpr int kEpiSlots = 2;
constexpr int kNsSmemBytes =
    kStages * (kAStageBytes + kBStageBytes) + kEpiSlots * kEpiSlotBytes + 1024 /*align*/ + 256;
static_assert(kNsSmemBytes <= 232448, "exceeds the 227 KB of shared memory per block");
constexpr int kPThreads = 256;

enum { kModeMuon = 0, kModeOrtho = 1 };
// kSquare: P = b A + c A A over upper tiles (quintic coefficients), A symmetric.
enum { kSyrk = 0, kGemm = 1, kSquare = 2 };

// One matrix of a launch group.  X is the m x n "wide" view (m <= n) of the
// parameter: X = M when rows <= cols, X = M^T otherwise (T = 1), stored
// row-major with pitch ldx elements in scratch memory.
struct MatDesc {
  void* W;             // parameter (Muon) or in/out matrix (orthogonalise)
  const void* G;       // gradient (Muon) or input matrix (orthogonalise)
  float* buf;          // fp32 momentum buffer, or nullptr (orthogonalise)
  int64_t rows, cols;  // parameter shape
  int64_t ldx, lda;    // pitches (elements) of X and A
  void* X[2];          // ping-pong iterates
  void* Xop[2];        // tensor-core operand copies of X (tf32-rounded for fp32; == X for bf16)
  void* A;             // Gram matrix m x m
  void* P;             // quintic coefficients: b A + c A A (m x m, pitch lda), else nullptr
  float* scale;        // s = 1 / (||M||_F + 1e-7), written by finalize_kernel
  float lr_mult;       // per-matrix multiplier of lr (1 on the pages' update)
  int m, n, T;
  int mode;            // kModeMuon | kModeOrtho
  int g_bf16;          // gradient / input storage: 1 bf16, 0 fp32
  int vec4;            // parameter rows allow 4-element vector access
  int ptiles_c;        // transposed prologue tiles per parameter row band
  int b3d;             // xmn maps are 3-D (bf16, n % 64 == 0): one load brings a whole B operand
  int world;           // > 1: the gradient is the mean of `world` buffers Gr[0..world)
  const void* const* Gr;  // device array of the ranks' gradient buffers (rank order), or nullptr
  int tmaps;           // the gt / bt tensor maps bring a transposed prologue item's G and buf
  int a3d;             // amn3 exists (bf16, m % 64 == 0): one load per transposed SQUARE operand
};

struct alignas(64) MatMaps {
  CUtensorMap xk[2];   // Xop as K-major operand, box (128 B of K) x 128 rows
  CUtensorMap xkw[2];  // same, box (128 B of K) x 256 rows: a whole SYRK B operand in one load
  CUtensorMap xmn[2];  // Xop as MN-major operand, box (128 B of N) x (BK rows of K); with b3d a
                       // 3-D view {64 columns, rows, column blocks of 64} and a box of 4 blocks
  CUtensorMap a;       // A as K-major operand, box (128 B of K) x 128 rows
  CUtensorMap aw;      // A, box (128 B of K) x 256 rows: the B operand of A A in one load
  CUtensorMap p;       // P as K-major operand (the GEMM's A operand in quintic mode)
  CUtensorMap amn;     // A as MN-major operand, box (128 B of M) x (BK rows of K): the GEMM
  CUtensorMap pmn;     // reads A's (or P's) lower k-blocks transposed from the upper triangle
  CUtensorMap xmn2[2]; // with b3d: the 3-D view of xmn with a box of 2 blocks (128 columns),
                       // one CTA's half of the B operand of a pair GEMM tile
  CUtensorMap amn3[2]; // with a3d: A as a 3-D MN-major view {64 columns, rows, column blocks}
                       // (as xmn), boxes of 4 and 2 blocks: a 256- or 128-row transposed
                       // operand of the SQUARE stage
  CUtensorMap gt;      // with tmaps: G (rows x cols) and buf, box kTC columns x kTR rows, no
  CUtensorMap bt;      // swizzle; their addresses follow the caller's through patch_kernel
};

struct NsParams {
  const MatDesc* mats;
  const MatMaps* maps;
  const int* order;        // matrix index for each position (longest K first)
  const int* tile_prefix;  // [nmat + 1] tile offsets in that order
  int nmat;
  int ntiles;
  int cur;                 // X buffer holding the current iterate
  int first;               // fold s into this stage (first NS step)
  int last;                // GEMM writes the final result (last NS step)
  float lr, wd;            // update scalars (used when last)
  float ca, cb;            // GEMM: X <- ca X + cb (A or P) X; SQUARE: P = cb A + cc A A
  float cc;
  int quintic;             // GEMM reads P instead of A
  int mirror;              // SYRK / SQUARE: also write the lower triangle (A^T of the upper)
  int a_upper;             // GEMM: A (or P) holds its upper triangle and the diagonal 128-blocks
                           // only; the k-blocks left of the diagonal block are read transposed.
                           // SQUARE: A holds its upper triangle and whole diagonal 256-blocks;
                           // both operands read their k-blocks left of that block transposed
  int diag_full;           // SYRK with 256 x 256 tiles, SQUARE: also store the lower-left
                           // 128 x 128 quarter of each diagonal 256-block (the pair GEMM reads
                           // the whole diagonal 256-block K-major)
  int* err;                // device error word
  uint64_t wait_limit_ns;
};

struct ElemParams {
  const MatDesc* mats;
  const int64_t* ptile_prefix;  // [nmat + 1] prologue tile offsets
  float* partials;              // one partial sum of squares per prologue tile
  int nmat;
  int64_t ntiles;
  float mu;
  int nesterov;
  float lr, wd;                 // apply_kernel only
  const float* clip;            // gradient scale (global-norm clipping) or nullptr
  double* gpartials;            // grad_norm_kernel: one partial sum of g^2 per item
  int* err;                     // prologue_tma_kernel: device error word and bound of its waits
  uint64_t wait_limit_ns;
  const MatMaps* maps;          // prologue_tma_kernel: the matrices' gt / bt maps
};

// ------------------------------------------------------------------ helpers
template <typename E> __device__ __forceinline__ float to_f(E v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <typename E> __device__ __forceinline__ E from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Value as stored for use as a tensor-core operand: bf16 storage rounds by
// itself; fp32 operands are pre-rounded to tf32 (nearest) so that the
// MMA's own truncation of the low mantissa bits is exact.
template <typename E> __device__ __forceinline__ float op_round(float v) {
  return sizeof(E) == 4 ? tf32_rna(v) : v;
}

// Load / store 32 consecutive elements (row segment, 16-byte aligned).
template <typename E> __device__ __forceinline__ void load32(const E* src, float (&x)[32]);
template <> __device__ __forceinline__ void load32<float>(const float* src, float (&x)[32]) {
  const float4* s = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float4 v = s[i];
    x[4 * i] = v.x; x[4 * i + 1] = v.y; x[4 * i + 2] = v.z; x[4 * i + 3] = v.w;
  }
}
template <>
__device__ __forceinline__ void load32<__nv_bfloat16>(const __nv_bfloat16* src, float (&x)[32]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 v = s[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat162 p = *reinterpret_cast<const __nv_bfloat162*>(&w[j]);
      float2 f = __bfloat1622float2(p);
      x[8 * i + 2 * j] = f.x;
      x[8 * i + 2 * j + 1] = f.y;
    }
  }
}
template <typename E> __device__ __forceinline__ void store32(E* dst, const float (&x)[32]);
template <> __device__ __forceinline__ void store32<float>(float* dst, const float (&x)[32]) {
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 8; ++i) d[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
}
template <>
__device__ __forceinline__ void store32<__nv_bfloat16>(__nv_bfloat16* dst, const float (&x)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat162 p = __floats2bfloat162_rn(x[8 * i + 2 * j], x[8 * i + 2 * j + 1]);
      w[j] = *reinterpret_cast<uint32_t*>(&p);
    }
    d[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

__device__ __forceinline__ int find_slot(const int* prefix, int n, int t) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(prefix + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}
__device__ __forceinline__ int find_slot64(const int64_t* prefix, int n, int64_t t) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(prefix + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace dmuon
#include "ns_stage.cuh"   // the Newton-Schulz stage kernel (depends on the types above)
#include "syrk256.cuh"    // the SYRK stage (256 x 256 tiles)
#include "gemm_pair.cuh"  // the GEMM stage on CTA pairs (256 x 256 tiles)
namespace dmuon {

// ======================================================================
// Prologue: momentum + Nesterov + sum of squares + copy of M into X.
// Work items: a matrix that is not transposed is streamed flat, kFlatChunk
// consecutive elements per item (X has the parameter's layout); a transposed
// matrix is cut into kTR x kTC parameter tiles that are transposed through
// shared memory.  One partial sum of squares per item.
// ======================================================================
constexpr int kFlatChunk = 8192;       // elements per flat item (256 threads x 4 x 8)
constexpr int kTR = 64, kTC = 128;     // transposed item: 64 parameter rows x 128 columns
// Dynamic shared memory of the prologue: the staged gradient (room for fp32)
// and momentum of one item; a transposed item reuses it as its 64 x 129
// fp32 transpose tile once every thread has read its staged inputs.
constexpr int kProStageG = kFlatChunk * 4;
constexpr int kProSmemBytes = kFlatChunk * 8;
static_assert(kTR * (kTC + 1) * 4 <= kProSmemBytes, "transpose tile must fit the staging area");

// Stage 8 consecutive input elements (one thread's segment) into shared
// memory with 16-byte asynchronous copies: the gradient at sg (2 or 4 bytes
// an element), the momentum at sb.  Only whole, 16-byte aligned segments.
template <bool kRanks>
__device__ __forceinline__ void stage8(const MatDesc& md, int64_t idx, bool has_buf, uint8_t* sg, float* sb) {
  if (kRanks && md.world > 1) {
    // the mean over the ranks is read directly at use
  } else if (md.g_bf16) {
    cp_async16(sg, reinterpret_cast<const __nv_bfloat16*>(md.G) + idx);
  } else {
    const float* g = reinterpret_cast<const float*>(md.G) + idx;
    cp_async16(sg, g);
    cp_async16(sg + 16, g + 4);
  }
  if (has_buf) {
    cp_async16(sb, md.buf + idx);
    cp_async16(sb + 4, md.buf + idx + 4);
  }
}
template <bool kRanks>
__device__ __forceinline__ void unstage8(const MatDesc& md, bool has_buf, const uint8_t* sg, const float* sb,
                                         float (&g)[8], float (&b)[8]) {
  if (kRanks && md.world > 1) {
    // not staged: the caller reads the mean over the ranks
  } else if (md.g_bf16) {
    const uint4 u = *reinterpret_cast<const uint4*>(sg);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
      g[2 * j] = f.x;
      g[2 * j + 1] = f.y;
    }
  } else {
    const float4 x = *reinterpret_cast<const float4*>(sg);
    const float4 y = *reinterpret_cast<const float4*>(sg + 16);
    g[0] = x.x; g[1] = x.y; g[2] = x.z; g[3] = x.w;
    g[4] = y.x; g[5] = y.y; g[6] = y.z; g[7] = y.w;
  }
  if (has_buf) {
    const float4 x = *reinterpret_cast<const float4*>(sb);
    const float4 y = *reinterpret_cast<const float4*>(sb + 4);
    b[0] = x.x; b[1] = x.y; b[2] = x.z; b[3] = x.w;
    b[4] = y.x; b[5] = y.y; b[6] = y.z; b[7] = y.w;
  }
}

// 8 consecutive elements (bf16 or fp32) of G, 16-byte aligned when vec.
__device__ __forceinline__ void load8_from(const void* G, int g_bf16, int64_t idx, bool vec, int valid,
                                           float (&g)[8]) {
  if (g_bf16) {
    const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(G) + idx;
    if (vec) {
      const uint4 u = *reinterpret_cast<const uint4*>(src);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
        g[2 * j] = f.x;
        g[2 * j + 1] = f.y;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) g[e] = (e < valid) ? __bfloat162float(src[e]) : 0.0f;
    }
  } else {
    const float* src = reinterpret_cast<const float*>(G) + idx;
    if (vec) {
      const float4 a = *reinterpret_cast<const float4*>(src);
      const float4 b = *reinterpret_cast<const float4*>(src + 4);
      g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w;
      g[4] = b.x; g[5] = b.y; g[6] = b.z; g[7] = b.w;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) g[e] = (e < valid) ? src[e] : 0.0f;
    }
  }
}
// 8 consecutive gradient elements.  With world > 1 the gradient is the
// data-parallel mean, read straight from every rank's buffer (in a multi-GPU
// job, peer memory mapped into this process): an fp32 sum in rank order,
// then one division by the number of ranks.  Kernels instantiated with
// kRanks = false (every launch without such matrices) compile this out and
// keep their register budget.
template <bool kRanks>
__device__ __forceinline__ void load8_in(const MatDesc& md, int64_t idx, bool vec, int valid, float (&g)[8]) {
  if (!kRanks || md.world <= 1) {
    load8_from(md.G, md.g_bf16, idx, vec, valid, g);
    return;
  }
  load8_from(md.Gr[0], md.g_bf16, idx, vec, valid, g);
  int r = 1;
  // Four ranks' loads in flight at once; the sum stays in rank order.
  for (; r + 3 < md.world; r += 4) {
    float h0[8], h1[8], h2[8], h3[8];
    load8_from(md.Gr[r], md.g_bf16, idx, vec, valid, h0);
    load8_from(md.Gr[r + 1], md.g_bf16, idx, vec, valid, h1);
    load8_from(md.Gr[r + 2], md.g_bf16, idx, vec, valid, h2);
    load8_from(md.Gr[r + 3], md.g_bf16, idx, vec, valid, h3);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      g[e] = __fadd_rn(__fadd_rn(__fadd_rn(__fadd_rn(g[e], h0[e]), h1[e]), h2[e]), h3[e]);
  }
  for (; r < md.world; ++r) {
    float h[8];
    load8_from(md.Gr[r], md.g_bf16, idx, vec, valid, h);
#pragma unroll
    for (int e = 0; e < 8; ++e) g[e] = __fadd_rn(g[e], h[e]);
  }
  const float w = static_cast<float>(md.world);
#pragma unroll
  for (int e = 0; e < 8; ++e) g[e] = __fdiv_rn(g[e], w);
}
__device__ __forceinline__ void load8_f32(const float* src, bool vec, int valid, float (&b)[8]) {
  if (vec) {
    const float4 x = *reinterpret_cast<const float4*>(src);
    const float4 y = *reinterpret_cast<const float4*>(src + 4);
    b[0] = x.x; b[1] = x.y; b[2] = x.z; b[3] = x.w;
    b[4] = y.x; b[5] = y.y; b[6] = y.z; b[7] = y.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) b[e] = (e < valid) ? src[e] : 0.0f;
  }
}
__device__ __forceinline__ void store8_f32(float* dst, bool vec, int valid, const float (&b)[8]) {
  if (vec) {
    *reinterpret_cast<float4*>(dst) = make_float4(b[0], b[1], b[2], b[3]);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(b[4], b[5], b[6], b[7]);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (e < valid) dst[e] = b[e];
  }
}
// 8 consecutive X elements (16-byte aligned when vec).
template <typename E>
__device__ __forceinline__ void store8_x(E* dst, bool vec, int valid, const float (&v)[8]) {
  if (vec && sizeof(E) == 2) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
      w[j] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if (vec) {
    float* d = reinterpret_cast<float*>(dst);
    *reinterpret_cast<float4*>(d) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(d + 4) = make_float4(v[4], v[5], v[6], v[7]);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (e < valid) dst[e] = from_f<E>(v[e]);
  }
}

// Momentum / Nesterov on N values; returns M, updates b in place.  With
// gradient clipping the gradient enters as fl32(g * c).
template <int N>
__device__ __forceinline__ void momentum_n(const ElemParams& p, bool has_buf, float (&g)[N],
                                           float (&b)[N], float (&M)[N]) {
  if (p.clip != nullptr) {
    const float c = *p.clip;
#pragma unroll
    for (int e = 0; e < N; ++e) g[e] = __fmul_rn(g[e], c);
  }
#pragma unroll
  for (int e = 0; e < N; ++e) {
    if (has_buf) {
      // buf <- fl(fl(mu * buf) + g): two roundings, never fused.
      b[e] = __fadd_rn(__fmul_rn(p.mu, b[e]), g[e]);
      M[e] = p.nesterov ? fmaf(p.mu, b[e], g[e]) : b[e];
    } else {
      M[e] = g[e];
    }
  }
}
__device__ __forceinline__ void momentum8(const ElemParams& p, bool has_buf, float (&g)[8],
                                          float (&b)[8], float (&M)[8]) {
  momentum_n<8>(p, has_buf, g, b, M);
}

template <typename E, bool kRanks>
__device__ __forceinline__ float prologue_flat(const ElemParams& p, const MatDesc& md, int64_t item,
                                               uint8_t* stage) {
  const int tid = threadIdx.x;
  const int64_t numel = md.rows * md.cols;
  const int64_t e_begin = item * kFlatChunk;
  const bool has_buf = md.buf != nullptr;
  const bool flat_x = (md.ldx == md.cols);
  E* X = reinterpret_cast<E*>(md.X[0]);
  E* Xo = reinterpret_cast<E*>(md.Xop[0]);
  const int gb = md.g_bf16 ? 2 : 4;
  float* sbuf = reinterpret_cast<float*>(stage + kProStageG);
  // Four rounds of 8 consecutive elements per thread.  The whole, aligned
  // segments of all four rounds are staged into shared memory first, so
  // 4 x (8 g + 8 buf) elements per thread are in flight at once; each thread
  // reads back only what it staged itself.
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int le = (j * kPThreads + tid) * 8;
    const int64_t e = e_begin + le;
    if (md.vec4 && e + 8 <= numel) stage8<kRanks>(md, e, has_buf, stage + le * gb, sbuf + le);
  }
  cp_async_commit();
  cp_async_wait_all();
  float ss = 0.0f;
#pragma unroll 1
  for (int j = 0; j < 4; ++j) {
    const int le = (j * kPThreads + tid) * 8;
    const int64_t e = e_begin + le;
    if (e >= numel) break;
    const int valid = static_cast<int>(numel - e < 8 ? numel - e : 8);
    const bool vec = md.vec4 && valid == 8;
    float g[8], b[8], M[8];
    if (vec) {
      unstage8<kRanks>(md, has_buf, stage + le * gb, sbuf + le, g, b);
      if (kRanks && md.world > 1) load8_in<kRanks>(md, e, true, 8, g);
    } else {
      load8_in<kRanks>(md, e, vec, valid, g);
      if (has_buf) load8_f32(md.buf + e, vec, valid, b);
    }
    momentum8(p, has_buf, g, b, M);
    if (has_buf) store8_f32(md.buf + e, vec, valid, b);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k >= valid) M[k] = 0.0f;
      ss = fmaf(M[k], M[k], ss);
    }
    if (flat_x) {
      store8_x<E>(X + e, valid == 8, valid, M);
      if (sizeof(E) == 4 && Xo != X) {
#pragma unroll
        for (int k = 0; k < 8; ++k) M[k] = op_round<E>(M[k]);
        store8_x<E>(Xo + e, valid == 8, valid, M);
      }
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (k < valid) {
          const int64_t r = (e + k) / md.cols, c = (e + k) - r * md.cols;
          X[r * md.ldx + c] = from_f<E>(M[k]);
          if (sizeof(E) == 4 && Xo != X) Xo[r * md.ldx + c] = from_f<E>(op_round<E>(M[k]));
        }
      }
    }
  }
  return ss;
}

template <typename E, bool kRanks>
__device__ __forceinline__ float prologue_transposed(const ElemParams& p, const MatDesc& md, int64_t item,
                                                     uint8_t* stage) {
  const int tid = threadIdx.x;
  const int ty = tid >> 4;      // 0..15: parameter rows ty + 16 i
  const int tx = tid & 15;      // 0..15: 8 consecutive parameter columns
  const int64_t tr = item / md.ptiles_c, tc = item - tr * md.ptiles_c;
  const int64_t r0 = tr * kTR, c0 = tc * kTC;
  const int64_t rows = md.rows, cols = md.cols;
  const bool has_buf = md.buf != nullptr;
  const int64_t c = c0 + tx * 8;
  const int gb = md.g_bf16 ? 2 : 4;
  float* sbuf = reinterpret_cast<float*>(stage + kProStageG);
  // Stage this thread's four row segments (whole, aligned ones) first.
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = r0 + ty + 16 * i;
    const int64_t idx = r * cols + c;
    const int slot = (i * kPThreads + tid) * 8;
    if (md.vec4 && r < rows && c + 8 <= cols && (idx & 7) == 0)
      stage8<kRanks>(md, idx, has_buf, stage + slot * gb, sbuf + slot);
  }
  cp_async_commit();
  cp_async_wait_all();
  float Mv[4][8];
  float ss = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = r0 + ty + 16 * i;
    const int valid = (r < rows && c < cols) ? static_cast<int>(cols - c < 8 ? cols - c : 8) : 0;
    float g[8], b[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) { g[k] = 0.0f; b[k] = 0.0f; }
    const int64_t idx = r * cols + c;
    const bool vec = md.vec4 && valid == 8 && ((idx & 7) == 0);
    if (vec) {
      const int slot = (i * kPThreads + tid) * 8;
      unstage8<kRanks>(md, has_buf, stage + slot * gb, sbuf + slot, g, b);
      if (kRanks && md.world > 1) load8_in<kRanks>(md, idx, true, 8, g);
    } else if (valid > 0) {
      load8_in<kRanks>(md, idx, vec, valid, g);
      if (has_buf) load8_f32(md.buf + idx, vec, valid, b);
    }
    momentum8(p, has_buf, g, b, Mv[i]);
    if (valid > 0 && has_buf) store8_f32(md.buf + idx, vec, valid, b);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k >= valid) Mv[i][k] = 0.0f;
      ss = fmaf(Mv[i][k], Mv[i][k], ss);
    }
  }
  // Every thread has read its staged inputs: the area becomes the transpose tile.
  __syncthreads();
  float (*sM)[kTC + 1] = reinterpret_cast<float (*)[kTC + 1]>(stage);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int k = 0; k < 8; ++k) sM[ty + 16 * i][tx * 8 + k] = Mv[i][k];
  __syncthreads();
  // X row = parameter column (128 of them), X columns = the 64 parameter rows.
  E* X = reinterpret_cast<E*>(md.X[0]);
  E* Xo = reinterpret_cast<E*>(md.Xop[0]);
  const int xc8 = tid & 7;      // 8 threads x 8 elements = the 64 rows
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int cc = (tid >> 3) + 32 * pass;   // parameter column within the tile
    const int64_t xr = c0 + cc;
    const int64_t xc = r0 + xc8 * 8;
    if (xr < cols && xc < rows) {
      const int valid = (rows - xc >= 8) ? 8 : static_cast<int>(rows - xc);
      float v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = sM[xc8 * 8 + k][cc];
      store8_x<E>(X + xr * md.ldx + xc, valid == 8, valid, v);
      if (sizeof(E) == 4 && Xo != X) {
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = op_round<E>(v[k]);
        store8_x<E>(Xo + xr * md.ldx + xc, valid == 8, valid, v);
      }
    }
  }
  __syncthreads();
  return ss;
}

template <typename E, bool kRanks = false>
__global__ void __launch_bounds__(kPThreads) prologue_kernel(const __grid_constant__ ElemParams p) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ __align__(128) uint8_t pro_stage[];   // kProSmemBytes
  __shared__ float red[kPThreads / 32];
  const int tid = threadIdx.x;
  // A block's items only move forward through the matrices: one search,
  // then a cursor.
  int mi = blockIdx.x < p.ntiles ? find_slot64(p.ptile_prefix, p.nmat, blockIdx.x) : 0;
  for (int64_t t = blockIdx.x; t < p.ntiles; t += gridDim.x) {
    while (t >= __ldg(p.ptile_prefix + mi + 1)) ++mi;
    const MatDesc& md = p.mats[mi];
    const int64_t item = t - __ldg(p.ptile_prefix + mi);
    float ss = md.T ? prologue_transposed<E, kRanks>(p, md, item, pro_stage)
                    : prologue_flat<E, kRanks>(p, md, item, pro_stage);
    // Fixed-order block reduction of the item's sum of squares.
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    __syncthreads();
    if (tid == 0) {
      float acc = 0.0f;
#pragma unroll
      for (int w = 0; w < kPThreads / 32; ++w) acc += red[w];
      p.partials[t] = acc;
    }
    __syncthreads();
  }
}

// ======================================================================
// Pipelined prologue for bf16 iterates and one gradient buffer per matrix.
// The same work items as prologue_kernel.  A producer warp streams each
// item's gradient and momentum into a ring of shared-memory stages with bulk
// asynchronous copies (two for a flat item, two per parameter row of a
// transposed item) while eight consumer warps work on an earlier stage, so
// the loads stay in flight across items instead of being issued and awaited
// one item at a time.  A transposed item is mapped so that each consumer
// thread owns 8 parameter rows x 4 columns: its four X row segments (8
// consecutive parameter rows of one column, 16 bytes) are stored straight to
// global memory, without a shared-memory transpose.  Items that are not
// whole and 16-byte aligned (a matrix's ragged edge) are read from global
// memory directly by the consumers.
// ======================================================================
constexpr int kPtConsumers = 256;                 // 8 consumer warps
constexpr int kPtThreads = kPtConsumers + 32;     // + 1 producer warp
template <bool kGBf16> struct PtCfg {
  static constexpr int kGBytes = kFlatChunk * (kGBf16 ? 2 : 4);   // an item's gradient
  static constexpr int kBBytes = kFlatChunk * 4;                   // an item's momentum
  static constexpr int kStageBytes = kGBytes + kBBytes;
  static constexpr int kStages = kGBf16 ? 2 : 3;                   // 2 blocks / SM for bf16 gradients
  static constexpr int kBlocksPerSm = kGBf16 ? 2 : 1;
  static constexpr int kSmem = kStages * kStageBytes + 128 /*align*/;
};
static_assert(kTR * kTC == kFlatChunk, "a transposed item fills one stage like a flat item");
static_assert(PtCfg<false>::kSmem <= 232448 - 1024, "prologue stages exceed shared memory");
static_assert(2 * (PtCfg<true>::kSmem + 1024 + 256) <= 233472, "two bf16 prologue blocks must fit an SM");

// Whether an item's inputs come through the staged ring: whole items of
// matrices whose rows start on 16-byte boundaries.
__device__ __forceinline__ bool pt_whole(const MatDesc& md, int64_t item) {
  if (!md.vec4) return false;
  if (!md.T) return (item + 1) * kFlatChunk <= md.rows * md.cols;
  const int64_t tr = item / md.ptiles_c, tc = item - tr * md.ptiles_c;
  return (md.cols % 8 == 0) && (tr + 1) * kTR <= md.rows && (tc + 1) * kTC <= md.cols;
}

// Flat item: thread `ct` handles the same 4 x 8 elements as prologue_flat,
// with the same arithmetic and summation order.
__device__ __forceinline__ float pt_flat(const ElemParams& p, const MatDesc& md, int64_t item, bool whole,
                                         const uint8_t* sg, const float* sb, int ct) {
  const int64_t numel = md.rows * md.cols;
  const int64_t e_begin = item * kFlatChunk;
  const bool has_buf = md.buf != nullptr;
  const bool flat_x = (md.ldx == md.cols);
  const int gb = md.g_bf16 ? 2 : 4;
  __nv_bfloat16* X = reinterpret_cast<__nv_bfloat16*>(md.X[0]);
  float ss = 0.0f;
#pragma unroll 1
  for (int j = 0; j < 4; ++j) {
    const int le = (j * kPtConsumers + ct) * 8;
    const int64_t e = e_begin + le;
    if (e >= numel) break;
    const int valid = static_cast<int>(numel - e < 8 ? numel - e : 8);
    const bool vec = md.vec4 && valid == 8;
    float g[8], b[8], M[8];
    if (whole) {
      unstage8<false>(md, has_buf, sg + le * gb, sb + le, g, b);
    } else {
      load8_in<false>(md, e, vec, valid, g);
      if (has_buf) load8_f32(md.buf + e, vec, valid, b);
    }
    momentum8(p, has_buf, g, b, M);
    if (has_buf) store8_f32(md.buf + e, vec, valid, b);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k >= valid) M[k] = 0.0f;
      ss = fmaf(M[k], M[k], ss);
    }
    if (flat_x) {
      store8_x<__nv_bfloat16>(X + e, valid == 8, valid, M);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (k < valid) {
          const int64_t r = (e + k) / md.cols, c = (e + k) - r * md.cols;
          X[r * md.ldx + c] = __float2bfloat16_rn(M[k]);
        }
      }
    }
  }
  return ss;
}

// Transposed item (kTR parameter rows x kTC columns): thread `ct` owns rows
// rb*8 .. rb*8+7 and columns cg*4 .. cg*4+3 of the item.  Within a warp the
// 8 column groups x 4 row blocks read 128 contiguous bytes of momentum per
// staged row (no bank conflicts) and write 64-byte runs of 8 X rows.
constexpr int kPtRB = kTR / 8, kPtCG = kTC / 4;   // row blocks and column groups of an item
static_assert(kPtRB * kPtCG == kPtConsumers && kPtRB % 4 == 0 && kPtCG % 8 == 0,
              "transposed item mapping: 4 row blocks x 8 column groups per warp");
__device__ __forceinline__ float pt_transposed(const ElemParams& p, const MatDesc& md, int64_t item, bool whole,
                                               const uint8_t* sg, const float* sb, int ct) {
  const int w = ct >> 5, l = ct & 31;
  const int rb = (l >> 3) + 4 * (w % (kPtRB / 4));
  const int cg = (l & 7) + 8 * (w / (kPtRB / 4));
  const int64_t tr = item / md.ptiles_c, tc = item - tr * md.ptiles_c;
  const int64_t r0 = tr * kTR, c0 = tc * kTC;
  const int64_t rows = md.rows, cols = md.cols;
  const bool has_buf = md.buf != nullptr;
  const int lc = cg * 4;
  const int64_t c = c0 + lc;
  float Mv[8][4];
  float ss = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int lr = rb * 8 + j;
    const int64_t r = r0 + lr;
    float g[4], b[4];
    int valid = 4;
    if (whole) {
      if (md.g_bf16) {
        const uint2 u = *reinterpret_cast<const uint2*>(sg + (lr * kTC + lc) * 2);
        const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        g[0] = f0.x; g[1] = f0.y; g[2] = f1.x; g[3] = f1.y;
      } else {
        const float4 v = *reinterpret_cast<const float4*>(sg + (lr * kTC + lc) * 4);
        g[0] = v.x; g[1] = v.y; g[2] = v.z; g[3] = v.w;
      }
      if (has_buf) {
        const float4 v = *reinterpret_cast<const float4*>(sb + lr * kTC + lc);
        b[0] = v.x; b[1] = v.y; b[2] = v.z; b[3] = v.w;
      }
    } else {
      valid = (r < rows && c < cols) ? static_cast<int>(cols - c < 4 ? cols - c : 4) : 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const bool in = k < valid;
        const int64_t idx = r * cols + c + k;
        g[k] = !in ? 0.0f
               : md.g_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(md.G)[idx])
                           : reinterpret_cast<const float*>(md.G)[idx];
        b[k] = (in && has_buf) ? md.buf[idx] : 0.0f;
      }
    }
    momentum_n<4>(p, has_buf, g, b, Mv[j]);
    if (has_buf) {
      float* dst = md.buf + r * cols + c;
      if (whole) {
        *reinterpret_cast<float4*>(dst) = make_float4(b[0], b[1], b[2], b[3]);
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (k < valid) dst[k] = b[k];
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (k >= valid) Mv[j][k] = 0.0f;
      ss = fmaf(Mv[j][k], Mv[j][k], ss);
    }
  }
  // X row = parameter column, X columns = parameter rows.
  __nv_bfloat16* X = reinterpret_cast<__nv_bfloat16*>(md.X[0]);
  const int64_t xc = r0 + rb * 8;
  const bool vec_x = whole && (md.ldx % 8 == 0);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int64_t xr = c + q;
    if (vec_x) {
      uint32_t u[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(Mv[2 * h][q], Mv[2 * h + 1][q]);
        u[h] = *reinterpret_cast<const uint32_t*>(&v);
      }
      *reinterpret_cast<uint4*>(X + xr * md.ldx + xc) = make_uint4(u[0], u[1], u[2], u[3]);
    } else if (xr < cols && xc < rows) {
      const int valid = (rows - xc >= 8) ? 8 : static_cast<int>(rows - xc);
#pragma unroll
      for (int h = 0; h < 8; ++h)
        if (h < valid) X[xr * md.ldx + xc + h] = __float2bfloat16_rn(Mv[h][q]);
    }
  }
  return ss;
}

template <bool kGBf16>
__global__ void __launch_bounds__(kPtThreads) prologue_tma_kernel(const __grid_constant__ ElemParams p) {
  griddep_wait();
  griddep_launch_dependents();
  using Cfg = PtCfg<kGBf16>;
  constexpr int S = Cfg::kStages;
  extern __shared__ __align__(128) uint8_t pt_raw[];    // Cfg::kSmem
  uint8_t* pt_smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pt_raw) + 127) &
                                                ~static_cast<uintptr_t>(127));
  __shared__ __align__(8) uint64_t full_bar[S];
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ float red[2][kPtConsumers / 32];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kPtConsumers / 32);
    }
    fence_mbar_init();
  }
  __syncthreads();
  int mi = blockIdx.x < p.ntiles ? find_slot64(p.ptile_prefix, p.nmat, blockIdx.x) : 0;
  if (warp == kPtConsumers / 32) {
    // ---------------------------------------------------------- producer
    uint32_t it = 0;
    bool ok = true;
    int fenced = -1;                 // matrix whose tensor maps lane 0 has acquired
    for (int64_t t = blockIdx.x; t < p.ntiles; t += gridDim.x, ++it) {
      while (t >= __ldg(p.ptile_prefix + mi + 1)) ++mi;
      const MatDesc& md = p.mats[mi];
      const int64_t item = t - __ldg(p.ptile_prefix + mi);
      const int s = static_cast<int>(it % S);
      if (it >= S && !mbar_wait(&empty_bar[s], ((it / S) & 1u) ^ 1u, p.err, p.wait_limit_ns)) {
        ok = false;
        break;
      }
      uint8_t* sg = pt_smem + s * Cfg::kStageBytes;
      float* sb = reinterpret_cast<float*>(sg + Cfg::kGBytes);
      const bool has_buf = md.buf != nullptr;
      const uint32_t gb = md.g_bf16 ? 2u : 4u;
      if (!pt_whole(md, item)) {
        if (lane == 0) mbar_arrive(&full_bar[s]);
        continue;
      }
      if (!md.T) {
        if (lane == 0) {
          const int64_t e = item * kFlatChunk;
          mbar_arrive_expect_tx(&full_bar[s], kFlatChunk * (gb + (has_buf ? 4u : 0u)));
          bulk_load(sg, static_cast<const uint8_t*>(md.G) + e * gb, kFlatChunk * gb, &full_bar[s]);
          if (has_buf) bulk_load(sb, md.buf + e, kFlatChunk * 4, &full_bar[s]);
        }
      } else if (md.tmaps) {
        // One 2-D tensor load each for the item's gradient and momentum.
        if (lane == 0) {
          const MatMaps& mp = p.maps[mi];
          if (mi != fenced) {
            tensormap_acquire_gpu(&mp.gt);
            if (has_buf) tensormap_acquire_gpu(&mp.bt);
            fenced = mi;
          }
          const int64_t tr = item / md.ptiles_c, tc = item - tr * md.ptiles_c;
          const int32_t x = static_cast<int32_t>(tc * kTC), y = static_cast<int32_t>(tr * kTR);
          mbar_arrive_expect_tx(&full_bar[s], kFlatChunk * (gb + (has_buf ? 4u : 0u)));
          tma_load_2d(sg, &mp.gt, &full_bar[s], x, y);
          if (has_buf) tma_load_2d(sb, &mp.bt, &full_bar[s], x, y);
        }
      } else {
        // One bulk copy per parameter row of the item.
        if (lane == 0) mbar_arrive_expect_tx(&full_bar[s], kFlatChunk * (gb + (has_buf ? 4u : 0u)));
        __syncwarp();
        const int64_t tr = item / md.ptiles_c, tc = item - tr * md.ptiles_c;
#pragma unroll
        for (int h = 0; h < kTR / 32; ++h) {
          const int lr = lane + 32 * h;
          const int64_t idx = (tr * kTR + lr) * md.cols + tc * kTC;
          bulk_load(sg + lr * kTC * gb, static_cast<const uint8_t*>(md.G) + idx * gb, kTC * gb, &full_bar[s]);
          if (has_buf) bulk_load(sb + lr * kTC, md.buf + idx, kTC * 4, &full_bar[s]);
        }
      }
    }
    // Before leaving after a failed wait, let the copies already issued land
    // (bounded): the phase of each stage's last use, if any.
    if (!ok) {
      for (int s = 0; s < S; ++s) {
        if (it > static_cast<uint32_t>(s)) {
          const uint32_t last = it - 1 - ((it - 1 - s) % S);   // last iteration that used stage s
          mbar_wait(&full_bar[s], (last / S) & 1u, nullptr, p.wait_limit_ns);
        }
      }
    }
    return;
  }
  // ------------------------------------------------------------ consumers
  uint32_t it = 0;
  for (int64_t t = blockIdx.x; t < p.ntiles; t += gridDim.x, ++it) {
    while (t >= __ldg(p.ptile_prefix + mi + 1)) ++mi;
    const MatDesc& md = p.mats[mi];
    const int64_t item = t - __ldg(p.ptile_prefix + mi);
    const int s = static_cast<int>(it % S);
    // The consumers leave together, at the same item, if a wait gives up.
    const bool ok = mbar_wait(&full_bar[s], (it / S) & 1u, p.err, p.wait_limit_ns);
    if (!named_bar_and(2, kPtConsumers, ok)) break;
    const uint8_t* sg = pt_smem + s * Cfg::kStageBytes;
    const float* sb = reinterpret_cast<const float*>(sg + Cfg::kGBytes);
    const bool whole = pt_whole(md, item);
    float ss = md.T ? pt_transposed(p, md, item, whole, sg, sb, tid) : pt_flat(p, md, item, whole, sg, sb, tid);
    // This warp has read its staged values: release the stage.
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);
    // Fixed-order reduction of the item's sum of squares over the eight
    // warps (red alternates between two rows, so the next item's writes never
    // race thread 0's read of this one).
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) red[it & 1u][warp] = ss;
    named_bar_sync(1, kPtConsumers);
    if (tid == 0) {
      float acc = 0.0f;
#pragma unroll
      for (int w = 0; w < kPtConsumers / 32; ++w) acc += red[it & 1u][w];
      p.partials[t] = acc;
    }
  }
}

// Sum of squares of the gradients (fp64 accumulation), one partial per
// prologue work item (the items cover every gradient element exactly once).
template <typename E, bool kRanks = false>
__global__ void __launch_bounds__(kPThreads) grad_norm_kernel(const __grid_constant__ ElemParams p) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ double red[kPThreads / 32];
  const int tid = threadIdx.x;
  // A block's items only move forward through the matrices: one search,
  // then a cursor.
  int mi = blockIdx.x < p.ntiles ? find_slot64(p.ptile_prefix, p.nmat, blockIdx.x) : 0;
  for (int64_t t = blockIdx.x; t < p.ntiles; t += gridDim.x) {
    while (t >= __ldg(p.ptile_prefix + mi + 1)) ++mi;
    const MatDesc& md = p.mats[mi];
    const int64_t item = t - __ldg(p.ptile_prefix + mi);
    double ss = 0.0;
    const int64_t rows = md.rows, cols = md.cols;
    if (!md.T) {
      const int64_t numel = rows * cols;
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        const int64_t e = item * kFlatChunk + (static_cast<int64_t>(j) * kPThreads + tid) * 8;
        if (e >= numel) break;
        const int valid = static_cast<int>(numel - e < 8 ? numel - e : 8);
        float g[8];
        load8_in<kRanks>(md, e, md.vec4 && valid == 8, valid, g);
#pragma unroll
        for (int k = 0; k < 8; ++k) ss += static_cast<double>(g[k]) * g[k];
      }
    } else {
      const int64_t tr = item / md.ptiles_c, tc = item - tr * md.ptiles_c;
      const int64_t c = tc * kTC + (tid & 15) * 8;
#pragma unroll 1
      for (int i = 0; i < 4; ++i) {
        const int64_t r = tr * kTR + (tid >> 4) + 16 * i;
        if (r >= rows || c >= cols) continue;
        const int valid = static_cast<int>(cols - c < 8 ? cols - c : 8);
        const int64_t idx = r * cols + c;
        float g[8];
        load8_in<kRanks>(md, idx, md.vec4 && valid == 8 && ((idx & 7) == 0), valid, g);
#pragma unroll
        for (int k = 0; k < 8; ++k) ss += static_cast<double>(g[k]) * g[k];
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    __syncthreads();
    if (tid == 0) {
      double acc = 0.0;
#pragma unroll
      for (int w = 0; w < kPThreads / 32; ++w) acc += red[w];
      p.gpartials[t] = acc;
    }
    __syncthreads();
  }
}

// Global-norm clipping coefficient over all gradients of a call (one block,
// fixed-order sums): c = min(1, max_norm / (||g|| + 1e-6)); optionally also
// the norm itself.
struct ClipParams {
  const double* part[2];   // per dtype group: partial sums of g^2
  int64_t count[2];
  float max_norm;
  float* coef;             // out: device scalar read by the prologue
  float* norm_out;         // out (optional): the gradient norm before clipping
};

__global__ void clip_coef_kernel(const __grid_constant__ ClipParams cp) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ double red[32];
  double acc = 0.0;
  for (int gi = 0; gi < 2; ++gi)
    for (int64_t i = threadIdx.x; i < cp.count[gi]; i += blockDim.x) acc += cp.part[gi][i];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) tot += red[w];
    const double nrm = sqrt(tot);
    const double c = static_cast<double>(cp.max_norm) / (nrm + 1e-6);
    *cp.coef = static_cast<float>(c < 1.0 ? c : 1.0);
    if (cp.norm_out) *cp.norm_out = static_cast<float>(nrm);
  }
}

// One warp per matrix: s = 1 / (sqrt(sum of partials) + 1e-7), summed in a
// fixed order (deterministic).
__global__ void finalize_kernel(const __grid_constant__ ElemParams p) {
  griddep_wait();
  griddep_launch_dependents();
  const int mi = blockIdx.x;
  const int lane = threadIdx.x;
  const int64_t b = p.ptile_prefix[mi], e = p.ptile_prefix[mi + 1];
  double acc = 0.0;
  for (int64_t i = b + lane; i < e; i += 32) acc += static_cast<double>(p.partials[i]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) *p.mats[mi].scale = static_cast<float>(1.0 / (sqrt(acc) + 1e-7));
}

// ns_steps == 0: the result is X0 = s M itself.  Same work items as the
// prologue.
template <typename E>
__global__ void __launch_bounds__(kPThreads) apply_kernel(const __grid_constant__ ElemParams p) {
  griddep_wait();
  griddep_launch_dependents();
  // A block's items only move forward through the matrices: one search,
  // then a cursor.
  int mi = blockIdx.x < p.ntiles ? find_slot64(p.ptile_prefix, p.nmat, blockIdx.x) : 0;
  for (int64_t t = blockIdx.x; t < p.ntiles; t += gridDim.x) {
    while (t >= __ldg(p.ptile_prefix + mi + 1)) ++mi;
    const MatDesc& md = p.mats[mi];
    const int64_t item = t - __ldg(p.ptile_prefix + mi);
    const float s = *md.scale;
    const float lr = p.lr * md.lr_mult;
    const float decay = 1.0f - lr * p.wd;
    const E* X = reinterpret_cast<const E*>(md.X[0]);
    E* W = reinterpret_cast<E*>(md.W);
    int64_t r0, c0, nr, nc;
    if (md.T) {
      const int64_t tr = item / md.ptiles_c, tc = item - tr * md.ptiles_c;
      r0 = tr * kTR; c0 = tc * kTC; nr = kTR; nc = kTC;
    } else {
      r0 = 0; c0 = item * kFlatChunk; nr = 1; nc = kFlatChunk;   // flat element range
    }
    for (int k = threadIdx.x; k < nr * nc; k += blockDim.x) {
      int64_t r, c;
      if (md.T) {
        r = r0 + k / nc; c = c0 + k % nc;
        if (r >= md.rows || c >= md.cols) continue;
      } else {
        const int64_t e = c0 + k;
        if (e >= md.rows * md.cols) continue;
        r = e / md.cols; c = e - r * md.cols;
      }
      const float x = s * to_f<E>(md.T ? X[c * md.ldx + r] : X[r * md.ldx + c]);
      E* wp = W + r * md.cols + c;
      if (md.mode == kModeOrtho) *wp = from_f<E>(x);
      else *wp = from_f<E>(fmaf(to_f<E>(*wp), decay, -lr * x));
    }
  }
}

// ======================================================================
// AdamW for the parameters that are not orthogonalised (the training
// guide's second group: biases, norms, embeddings, heads), all tensors of a
// call in one launch.  Per element, with c1 = fl32(1 - beta1),
// c2 = fl32(1 - beta2):
//   m <- fl(fl(beta1 m) + fl(c1 g))
//   v <- fl(fl(beta2 v) + fl(fl(c2 g) g))
//   p <- p (1 - lr wd) - (lr / bc1) m / (sqrt(v) / sqrt(bc2) + eps)
// with bc1 = 1 - beta1^t, bc2 = 1 - beta2^t (fp32 arithmetic for p).
// ======================================================================
constexpr int kAdamMaxTensors = 512;
constexpr int kAdamChunk = 8192;            // elements per work item (256 threads x 4 x 8)

struct AdamTensor {
  void* p;
  const void* g;
  float* m;
  float* v;
  int64_t numel;
  int64_t item0;     // first work item of this tensor
  int32_t p_bf16, g_bf16;
};

struct AdamParams {
  AdamTensor t[kAdamMaxTensors];
  int count;
  int64_t nitems;
  float b1, b2, c1, c2, eps, decay, step_size, inv_bc2_sqrt;
};

__device__ __forceinline__ void load8_any(const void* base, bool bf16, int64_t idx, bool vec, int valid,
                                          float (&x)[8]) {
  if (bf16) {
    const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(base) + idx;
    if (vec) {
      const uint4 u = *reinterpret_cast<const uint4*>(src);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
        x[2 * j] = f.x;
        x[2 * j + 1] = f.y;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = (e < valid) ? __bfloat162float(src[e]) : 0.0f;
    }
  } else {
    load8_f32(reinterpret_cast<const float*>(base) + idx, vec, valid, x);
  }
}

__global__ void __launch_bounds__(kPThreads) adamw_kernel(const __grid_constant__ AdamParams p) {
  griddep_wait();
  griddep_launch_dependents();
  for (int64_t it = blockIdx.x; it < p.nitems; it += gridDim.x) {
    int lo = 0, hi = p.count - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.t[mid].item0 <= it) lo = mid; else hi = mid - 1;
    }
    const AdamTensor& T = p.t[lo];
    const int64_t base = (it - T.item0) * kAdamChunk;
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
      const int64_t e = base + (static_cast<int64_t>(j) * kPThreads + threadIdx.x) * 8;
      if (e >= T.numel) break;
      const int valid = static_cast<int>(T.numel - e < 8 ? T.numel - e : 8);
      const bool vp = valid == 8 && ((reinterpret_cast<uintptr_t>(T.p) & 15) == 0);
      const bool vg = valid == 8 && ((reinterpret_cast<uintptr_t>(T.g) & 15) == 0);
      const bool vs = valid == 8 && ((reinterpret_cast<uintptr_t>(T.m) & 15) == 0) &&
                      ((reinterpret_cast<uintptr_t>(T.v) & 15) == 0);
      float g[8], m[8], v[8], w[8];
      load8_any(T.g, T.g_bf16, e, vg, valid, g);
      load8_f32(T.m + e, vs, valid, m);
      load8_f32(T.v + e, vs, valid, v);
      load8_any(T.p, T.p_bf16, e, vp, valid, w);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        m[k] = __fadd_rn(__fmul_rn(p.b1, m[k]), __fmul_rn(p.c1, g[k]));
        v[k] = __fadd_rn(__fmul_rn(p.b2, v[k]), __fmul_rn(__fmul_rn(p.c2, g[k]), g[k]));
        const float denom = __fadd_rn(__fmul_rn(__fsqrt_rn(v[k]), p.inv_bc2_sqrt), p.eps);
        w[k] = __fsub_rn(__fmul_rn(w[k], p.decay), __fmul_rn(p.step_size, __fdiv_rn(m[k], denom)));
      }
      store8_f32(T.m + e, vs, valid, m);
      store8_f32(T.v + e, vs, valid, v);
      if (T.p_bf16) store8_x<__nv_bfloat16>(reinterpret_cast<__nv_bfloat16*>(T.p) + e, vp, valid, w);
      else store8_f32(reinterpret_cast<float*>(T.p) + e, vp, valid, w);
    }
  }
}

// ======================================================================
// Clipping of several gradient segments, each with its own norm and
// coefficient (the training guide's fused regular / Muon / AdamW clipping,
// "梯度裁剪").  Three kernels:
//   clip_norm_kernel      one fp64 sum of squares per 32 KB work item (eight
//                         16-byte loads in flight per thread)
//   clip_finalize_kernel  one block per segment: fixed-order sum of its
//                         items, ||g||_s, c_s = fl32(min(1, max_s / (||g||_s + 1e-6)))
//   clip_scale_kernel     g <- fl32(g * c_s), rounded to the storage type,
//                         skipped for items of segments with c_s == 1
// The host sorts the tensors by segment, so each segment's items are one
// contiguous range.  The scale pass walks the items in reverse: the end of
// the norm pass is still in L2 when it starts.
// ======================================================================
constexpr int kClipMaxTensors = 512;     // tensors per launch (kernel parameter space)
constexpr int kClipMaxSegs = 64;
constexpr int kClipVecs = 8;             // 16-byte vectors per thread per work item, all in flight
constexpr int kClipItemBytes = kPThreads * kClipVecs * 16;   // 32 KB of gradient per work item

struct ClipTensor {
  void* g;
  int64_t numel;
  int64_t item0;     // first work item of this tensor (global numbering)
  int32_t seg;
  int32_t bf16;
};

struct ClipBucketParams {
  ClipTensor t[kClipMaxTensors];
  int count;            // tensors of this launch, in item order
  int64_t item_begin;   // global items [item_begin, item_end) of this launch
  int64_t item_end;
  double* partials;     // one per global item
  const float* coef;    // scale kernel: per-segment coefficient
};

struct ClipFinalizeParams {
  int64_t seg_item0[kClipMaxSegs + 1];
  float max_norm[kClipMaxSegs];
  const double* partials;
  float* coef;          // out: per-segment coefficient (scratch)
  float* norms_out;     // out (optional): per-segment norm before clipping
  float* coefs_out;     // out (optional): copy of the coefficients
};

__device__ __forceinline__ int clip_tensor_of(const ClipBucketParams& p, int64_t item) {
  int lo = 0, hi = p.count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.t[mid].item0 <= item) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Vector q of this thread in a work item: 16 bytes at byte offset
// item * 32 KB + (q * 256 + thread) * 16 of the tensor (consecutive threads,
// consecutive 16 bytes).  All kClipVecs vectors are loaded before any is used;
// a vector that is not whole, or of a tensor that is not 16-byte aligned, is
// read element by element, and elements past the tensor read as zero.
// `streaming`: the data is not read again soon (evict first from L2).
template <int EB, bool streaming>
__device__ __forceinline__ void clip_load(const ClipTensor& T, int64_t base_el, bool aligned16,
                                          uint4 (&v)[kClipVecs]) {
  constexpr int PER = 16 / EB;                 // elements per vector
#pragma unroll
  for (int q = 0; q < kClipVecs; ++q) {
    const int64_t e = base_el + static_cast<int64_t>(q * kPThreads + threadIdx.x) * PER;
    if (aligned16 && e + PER <= T.numel) {
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(T.g) + e * EB);
      v[q] = streaming ? __ldcs(src) : *src;
    } else {
      uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        if (e + k < T.numel) {
          if constexpr (EB == 2)
            w[k >> 1] |= static_cast<uint32_t>(static_cast<const uint16_t*>(T.g)[e + k]) << (16 * (k & 1));
          else
            w[k] = static_cast<const uint32_t*>(T.g)[e + k];
        }
      }
      v[q] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// Element k of a 16-byte vector as fp32 (bf16 widens exactly).
template <int EB>
__device__ __forceinline__ float clip_elem(const uint4& v, int k) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
  if constexpr (EB == 2) return __uint_as_float((k & 1) ? (u[k >> 1] & 0xFFFF0000u) : (u[k >> 1] << 16));
  else return __uint_as_float(u[k]);
}

template <int EB>
__device__ __forceinline__ double clip_sumsq(const ClipTensor& T, int64_t it) {
  constexpr int PER = 16 / EB;
  const int64_t base_el = (it - T.item0) * (kClipItemBytes / EB);
  uint4 v[kClipVecs];
  clip_load<EB, false>(T, base_el, (reinterpret_cast<uintptr_t>(T.g) & 15) == 0, v);
  double ss = 0.0;
#pragma unroll
  for (int q = 0; q < kClipVecs; ++q)
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const double x = static_cast<double>(clip_elem<EB>(v[q], k));
      ss = fma(x, x, ss);
    }
  return ss;
}

template <int EB>
__device__ __forceinline__ void clip_scale_item(const ClipTensor& T, int64_t it, float c) {
  constexpr int PER = 16 / EB;
  const int64_t base_el = (it - T.item0) * (kClipItemBytes / EB);
  const bool aligned16 = (reinterpret_cast<uintptr_t>(T.g) & 15) == 0;
  uint4 v[kClipVecs];
  clip_load<EB, true>(T, base_el, aligned16, v);
#pragma unroll
  for (int q = 0; q < kClipVecs; ++q) {
    const int64_t e = base_el + static_cast<int64_t>(q * kPThreads + threadIdx.x) * PER;
    if (e >= T.numel) continue;
    float y[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) y[k] = __fmul_rn(clip_elem<EB>(v[q], k), c);
    if (aligned16 && e + PER <= T.numel) {
      uint4 o;
      if constexpr (EB == 2) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          __nv_bfloat162 h = __floats2bfloat162_rn(y[2 * j], y[2 * j + 1]);
          w[j] = *reinterpret_cast<uint32_t*>(&h);
        }
        o = make_uint4(w[0], w[1], w[2], w[3]);
      } else {
        o = make_uint4(__float_as_uint(y[0]), __float_as_uint(y[1]), __float_as_uint(y[2]),
                       __float_as_uint(y[3]));
      }
      __stcs(reinterpret_cast<uint4*>(static_cast<uint8_t*>(T.g) + e * EB), o);
    } else {
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        if (e + k >= T.numel) break;
        if constexpr (EB == 2) static_cast<__nv_bfloat16*>(T.g)[e + k] = __float2bfloat16_rn(y[k]);
        else static_cast<float*>(T.g)[e + k] = y[k];
      }
    }
  }
}

__global__ void __launch_bounds__(kPThreads, 4) clip_norm_kernel(const __grid_constant__ ClipBucketParams p) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ double red[kPThreads / 32];
  const int tid = threadIdx.x;
  for (int64_t it = p.item_begin + blockIdx.x; it < p.item_end; it += gridDim.x) {
    const ClipTensor& T = p.t[clip_tensor_of(p, it)];
    double ss = T.bf16 ? clip_sumsq<2>(T, it) : clip_sumsq<4>(T, it);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    __syncthreads();
    if (tid == 0) {
      double acc = 0.0;
#pragma unroll
      for (int w = 0; w < kPThreads / 32; ++w) acc += red[w];
      p.partials[it] = acc;
    }
    __syncthreads();
  }
}

// One block of 1024 threads per segment; each thread keeps four running sums
// (four loads in flight) over a fixed stride, so the order is fixed.
constexpr int kClipFinThreads = 1024;
__global__ void __launch_bounds__(kClipFinThreads) clip_finalize_kernel(const __grid_constant__ ClipFinalizeParams p) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ double red[kClipFinThreads / 32];
  const int s = blockIdx.x;
  const int64_t b = p.seg_item0[s], e = p.seg_item0[s + 1];
  double a4[4] = {0.0, 0.0, 0.0, 0.0};
  int64_t i = b + threadIdx.x;
  for (; i + 3 * kClipFinThreads < e; i += 4 * kClipFinThreads) {
#pragma unroll
    for (int u = 0; u < 4; ++u) a4[u] += p.partials[i + u * kClipFinThreads];
  }
  for (int u = 0; i < e; i += kClipFinThreads, ++u) a4[u] += p.partials[i];
  double acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < kClipFinThreads / 32; ++w) tot += red[w];
    const double nrm = sqrt(tot);
    const double c = static_cast<double>(p.max_norm[s]) / (nrm + 1e-6);
    const float cf = static_cast<float>(c < 1.0 ? c : 1.0);   // a NaN norm gives 1
    p.coef[s] = cf;
    if (p.norms_out) p.norms_out[s] = static_cast<float>(nrm);
    if (p.coefs_out) p.coefs_out[s] = cf;
  }
}

__global__ void __launch_bounds__(kPThreads, 4) clip_scale_kernel(const __grid_constant__ ClipBucketParams p) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t n = p.item_end - p.item_begin;
  for (int64_t r = blockIdx.x; r < n; r += gridDim.x) {
    const int64_t it = p.item_end - 1 - r;
    const ClipTensor& T = p.t[clip_tensor_of(p, it)];
    const float c = p.coef[T.seg];
    if (c == 1.0f) continue;          // the identity: nothing to write
    if (T.bf16) clip_scale_item<2>(T, it, c);
    else clip_scale_item<4>(T, it, c);
  }
}

// ======================================================================
// Stream-ordered writes of library memory from kernel parameters (no host
// staging, no synchronous copy):
//   upload_kernel  copies up to kUploadWords 16-byte words (a launch plan:
//                  descriptors, tensor maps, tile tables) to device memory;
//                  the tensor maps among them are released to TMA.
//   patch_kernel   writes the caller's tensor addresses of one call into the
//                  matrix descriptors of a cached plan.
// ======================================================================
constexpr int kUploadWords = 1920;   // 30 KB of parameters
struct UploadParams {
  uint4* dst;
  int nwords;
  uint4 w[kUploadWords];
};
__global__ void __launch_bounds__(256) upload_kernel(const __grid_constant__ UploadParams p) {
  griddep_wait();
  griddep_launch_dependents();
  for (int i = threadIdx.x; i < p.nwords; i += blockDim.x) p.dst[i] = p.w[i];
  tensormap_release_gpu();
}

struct PatchEntry {
  void* W;
  const void* G;
  float* buf;
  int32_t index;    // matrix descriptor to patch
  int32_t vec4;
};
constexpr int kPatchMax = 480;        // entries per launch (about 15 KB of parameters)
struct PatchParams {
  MatDesc* mats;
  MatMaps* maps;
  int n;
  PatchEntry e[kPatchMax];
};
__global__ void __launch_bounds__(256) patch_kernel(const __grid_constant__ PatchParams p) {
  griddep_wait();
  griddep_launch_dependents();
  for (int i = threadIdx.x; i < p.n; i += blockDim.x) {
    MatDesc& d = p.mats[p.e[i].index];
    d.W = p.e[i].W;
    d.G = p.e[i].G;
    d.buf = p.e[i].buf;
    d.vec4 = p.e[i].vec4;
    // The prologue's G / buf tensor maps take the new addresses (used only
    // when the rows are 16-byte aligned, i.e. with vec4).
    if (d.tmaps && p.e[i].vec4) {
      MatMaps& mm = p.maps[p.e[i].index];
      tensormap_replace_address(&mm.gt, p.e[i].G);
      if (p.e[i].buf) tensormap_replace_address(&mm.bt, p.e[i].buf);
    }
  }
  tensormap_release_gpu();
}

// Test kernel: waits on a barrier that nothing arrives at; the bounded wait
// gives up after `limit_ns` and records kErrTimeout.
__global__ void wait_timeout_kernel(int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, err, limit_ns, 1024);
}

}  // namespace dmuon
