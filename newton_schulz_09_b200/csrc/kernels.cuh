// Kernels of the batched Muon update on sm_100a.
//
//   prologue_kernel     momentum, Nesterov input, per-tile sum of squares and
//                       the (transposed when rows > cols) copy of M into the
//                       iteration's X buffer.                     [HBM bound]
//   finalize_kernel     fixed-order sum of the tile partials per matrix and
//                       s = 1 / (||M||_F + 1e-7).
//   ns_stage_kernel     one Newton-Schulz stage for every matrix of a group
//                       in one persistent launch:
//                         SYRK  A = s^2 X X^T  (upper tiles, mirrored store)
//                         GEMM  X' = c (1.5 X - 0.5 A X), or on the last step
//                               the weight update / output write.   [tensor]
//   apply_kernel        the update for ns_steps == 0 (X = s M).
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
constexpr int kNsSmemBytes = kStages * (kAStageBytes + kBStageBytes) + 1024 /*align*/ + 256;
constexpr int kPT = 64;            // prologue tile: 64 x 64 parameter elements
constexpr int kPThreads = 256;

enum { kModeMuon = 0, kModeOrtho = 1 };
enum { kSyrk = 0, kGemm = 1 };

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
  float* scale;        // s = 1 / (||M||_F + 1e-7), written by finalize_kernel
  float lr_mult;       // per-matrix multiplier of lr (1 on the pages' update)
  int m, n, T;
  int mode;            // kModeMuon | kModeOrtho
  int g_bf16;          // gradient / input storage: 1 bf16, 0 fp32
  int vec4;            // parameter rows allow 4-element vector access
  int ptiles_c;        // prologue tiles per parameter row band
  int pad_;
};

struct alignas(64) MatMaps {
  CUtensorMap xk[2];   // Xop as K-major operand, box (128 B of K) x 128 rows
  CUtensorMap xmn[2];  // Xop as MN-major operand, box (128 B of N) x (BK rows of K)
  CUtensorMap a;       // A as K-major operand, box (128 B of K) x 128 rows
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

// Upper-triangle SYRK tiles of one matrix, enumerated column-band major:
// column band J (256 wide) holds row bands I = 0 .. 2J+1 (128 tall), so band
// J starts at J (J + 1).
__device__ __forceinline__ void syrk_tile_coords(int local, int& I, int& J) {
  int j = static_cast<int>((sqrtf(4.0f * static_cast<float>(local) + 1.0f) - 1.0f) * 0.5f);
  while ((j + 1) * (j + 2) <= local) ++j;
  while (j * (j + 1) > local) --j;
  J = j;
  I = local - j * (j + 1);
}

struct TileInfo {
  int mi, tm, tn, nkb;
};

template <int kMode, int BK>
__device__ __forceinline__ TileInfo decode_tile(const NsParams& p, int t) {
  TileInfo ti;
  const int slot = find_slot(p.tile_prefix, p.nmat, t);
  ti.mi = __ldg(p.order + slot);
  const int local = t - __ldg(p.tile_prefix + slot);
  const MatDesc& md = p.mats[ti.mi];
  if (kMode == kSyrk) {
    syrk_tile_coords(local, ti.tm, ti.tn);
    ti.nkb = (md.n + BK - 1) / BK;
  } else {
    const int nI = (md.m + kBM - 1) / kBM;
    ti.tn = local / nI;
    ti.tm = local - ti.tn * nI;
    ti.nkb = (md.m + BK - 1) / BK;
  }
  return ti;
}

// ======================================================================
// Newton-Schulz stage kernel (persistent, warp specialised).
// ======================================================================
template <int kMode, typename E>
__global__ void __launch_bounds__(kNsThreads, 1) ns_stage_kernel(const __grid_constant__ NsParams p) {
  constexpr int EB = static_cast<int>(sizeof(E));
  constexpr int BK = 128 / EB;              // K elements per stage (one 128-byte row)
  constexpr int MMA_K = 32 / EB;            // K per UMMA instruction
  constexpr int KSTEPS = BK / MMA_K;        // = 4
  constexpr uint32_t FMT = (EB == 2) ? 1u : 2u;
  constexpr uint32_t IDESC = make_idesc(FMT, 0u, kMode == kGemm ? 1u : 0u, kBM, kBN);
  constexpr int NBOX_B = (kMode == kGemm) ? kBN / BK : 2;
  constexpr uint32_t BOX_B_BYTES = (kMode == kGemm) ? BK * 128 : kAStageBytes;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sa = smem;
  uint8_t* sb = smem + kStages * kAStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sb + kStages * kBStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4 * 32);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  bool ok = true;
  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_phase[kStages];
    bool issued[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) { issued[s] = false; issued_phase[s] = 0; }
    for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x) {
      const TileInfo ti = decode_tile<kMode, BK>(p, t);
      const MatDesc& md = p.mats[ti.mi];
      const MatMaps& mp = p.maps[ti.mi];
      const CUtensorMap* mapA = (kMode == kSyrk) ? &mp.xk[p.cur] : &mp.a;
      const CUtensorMap* mapB = (kMode == kSyrk) ? &mp.xk[p.cur] : &mp.xmn[p.cur];
      int nb = 0;
      if (kMode == kSyrk) {
        nb = (ti.tn * kBN + 128 < md.m) ? 2 : 1;
      } else {
        const int left = md.n - ti.tn * kBN;
        nb = (left + BK - 1) / BK;
        if (nb > NBOX_B) nb = NBOX_B;
      }
      const uint32_t bytes = kAStageBytes + static_cast<uint32_t>(nb) * BOX_B_BYTES;
      for (int kb = 0; kb < ti.nkb; ++kb) {
        bool w = mbar_wait(&empty[stage], phase ^ 1u, p.err, p.wait_limit_ns);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[stage], bytes);
          uint8_t* a_dst = sa + stage * kAStageBytes;
          uint8_t* b_dst = sb + stage * kBStageBytes;
          tma_load_2d(a_dst, mapA, &full[stage], kb * BK, ti.tm * kBM);
          for (int j = 0; j < nb; ++j) {
            if (kMode == kSyrk)
              tma_load_2d(b_dst + j * kAStageBytes, mapB, &full[stage], kb * BK, ti.tn * kBN + j * 128);
            else
              tma_load_2d(b_dst + j * BOX_B_BYTES, mapB, &full[stage], ti.tn * kBN + j * BK, kb * BK);
          }
        }
        __syncwarp();
        issued[stage] = true;
        issued_phase[stage] = phase;
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok && lane == 0) {
      // Let every load already issued land before the CTA's memory goes away.
      for (int s = 0; s < kStages; ++s)
        if (issued[s]) mbar_wait(&full[s], issued_phase[s], nullptr, p.wait_limit_ns, 1024);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ UMMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int lt = 0;
    for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x, ++lt) {
      const TileInfo ti = decode_tile<kMode, BK>(p, t);
      const int b = lt & 1;
      const uint32_t tph = (static_cast<uint32_t>(lt) >> 1) & 1u;
      bool w = mbar_wait(&tempty[b], tph ^ 1u, p.err, p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * kBN);
      for (int kb = 0; kb < ti.nkb; ++kb) {
        w = mbar_wait(&full[stage], phase, p.err, p.wait_limit_ns);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_base = smem_u32(sa + stage * kAStageBytes);
          const uint32_t b_base = smem_u32(sb + stage * kBStageBytes);
#pragma unroll
          for (int k = 0; k < KSTEPS; ++k) {
            const uint64_t ad = sw128_desc(a_base + k * 32, 16, 1024);
            // MN-major B: 16-bit operands use the 16-byte-unit swizzle (8-line
            // K groups); 32-bit operands must use 32-byte units (4-line groups).
            const uint64_t bd =
                (kMode == kSyrk)
                    ? sw128_desc(b_base + k * 32, 16, 1024)
                    : sw128_desc(b_base + k * MMA_K * 128, BK * 128, EB == 2 ? 1024 : 512,
                                 EB == 2 ? kSwizzle128B : kSwizzle128B32);
            const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
            if (EB == 2) umma_f16(d_tmem, ad, bd, IDESC, acc);
            else umma_tf32(d_tmem, ad, bd, IDESC, acc);
          }
          umma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&tfull[b]);
      __syncwarp();
    }
    if (!ok && lane == 0) {
      // Wait for every UMMA this thread issued before TMEM is released.
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.wait_limit_ns, 1024);
    }
  } else {
    // ------------------------------------------------ epilogue (4 warps)
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int row_in_tile = q * 32 + lane;
    int lt = 0;
    for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x, ++lt) {
      const TileInfo ti = decode_tile<kMode, BK>(p, t);
      const MatDesc& md = p.mats[ti.mi];
      const int b = lt & 1;
      const uint32_t tph = (static_cast<uint32_t>(lt) >> 1) & 1u;
      const float s = *md.scale;
      bool w = mbar_wait(&tfull[b], tph, p.err, p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b * kBN);
      const int R = ti.tm * kBM + row_in_tile;
      const int m = md.m, n = md.n;
      if (kMode == kSyrk) {
        const float alpha = p.first ? s * s : 1.0f;
        E* A = reinterpret_cast<E*>(md.A);
        const int64_t lda = md.lda;
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_ld_wait();
          const int C0 = ti.tn * kBN + c * 32;
          if (R < m && C0 < m && C0 + 31 >= R) {
            float y[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) y[j] = op_round<E>(alpha * __uint_as_float(v[j]));
            E* arow = A + static_cast<int64_t>(R) * lda;
            if (C0 >= R && C0 + 32 <= m) {
              store32<E>(arow + C0, y);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int C = C0 + j;
                if (C < m && C >= R) arow[C] = from_f<E>(y[j]);
              }
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int C = C0 + j;
              if (C < m && C > R) A[static_cast<int64_t>(C) * lda + R] = from_f<E>(y[j]);
            }
          }
        }
      } else {
        const float cs = p.first ? s : 1.0f;
        const E* Xc = reinterpret_cast<const E*>(md.X[p.cur]);
        E* Xn = reinterpret_cast<E*>(md.X[p.cur ^ 1]);
        const int64_t ldx = md.ldx;
        const float lr = p.lr * md.lr_mult;
        const float decay = 1.0f - lr * p.wd;
        E* W = reinterpret_cast<E*>(md.W);
        const int64_t cols = md.cols;
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_ld_wait();
          const int C0 = ti.tn * kBN + c * 32;
          if (R < m && C0 < n) {
            const bool full_chunk = (C0 + 32 <= n);
            float x[32];
            const E* xrow = Xc + static_cast<int64_t>(R) * ldx + C0;
            if (full_chunk) {
              load32<E>(xrow, x);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) x[j] = (C0 + j < n) ? to_f<E>(xrow[j]) : 0.0f;
            }
            float y[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) y[j] = cs * (1.5f * x[j] - 0.5f * __uint_as_float(v[j]));
            if (!p.last) {
              E* dst = Xn + static_cast<int64_t>(R) * ldx + C0;
              if (full_chunk) {
                store32<E>(dst, y);
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (C0 + j < n) dst[j] = from_f<E>(y[j]);
              }
              if (EB == 4) {
                E* odst = reinterpret_cast<E*>(md.Xop[p.cur ^ 1]) + static_cast<int64_t>(R) * ldx + C0;
                float yr[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) yr[j] = op_round<E>(y[j]);
                if (full_chunk) {
                  store32<E>(odst, yr);
                } else {
#pragma unroll
                  for (int j = 0; j < 32; ++j)
                    if (C0 + j < n) odst[j] = from_f<E>(yr[j]);
                }
              }
            } else if (!md.T) {
              E* wrow = W + static_cast<int64_t>(R) * cols + C0;
              if (md.mode == kModeOrtho) {
                if (full_chunk && md.vec4 && (cols % (16 / EB) == 0)) {
                  store32<E>(wrow, y);
                } else {
#pragma unroll
                  for (int j = 0; j < 32; ++j)
                    if (C0 + j < n) wrow[j] = from_f<E>(y[j]);
                }
              } else {
                if (full_chunk && md.vec4 && (cols % (16 / EB) == 0)) {
                  float wv[32];
                  load32<E>(wrow, wv);
#pragma unroll
                  for (int j = 0; j < 32; ++j) wv[j] = fmaf(wv[j], decay, -lr * y[j]);
                  store32<E>(wrow, wv);
                } else {
#pragma unroll
                  for (int j = 0; j < 32; ++j)
                    if (C0 + j < n) wrow[j] = from_f<E>(fmaf(to_f<E>(wrow[j]), decay, -lr * y[j]));
                }
              }
            } else {
              // Transposed parameter: X[R][C] is W[C][R]; a warp's lanes hold
              // consecutive R, so each j writes one contiguous run.
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int C = C0 + j;
                if (C < n) {
                  E* wp = W + static_cast<int64_t>(C) * cols + R;
                  if (md.mode == kModeOrtho) *wp = from_f<E>(y[j]);
                  else *wp = from_f<E>(fmaf(to_f<E>(*wp), decay, -lr * y[j]));
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[b]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ======================================================================
// Prologue: momentum + Nesterov + sum of squares + copy into X (transposed
// when rows > cols).  One 64 x 64 parameter tile per iteration.
// ======================================================================
template <typename E>
__device__ __forceinline__ void load4_in(const MatDesc& md, int64_t idx, bool vec, int valid,
                                         float (&g)[4]) {
  if (md.g_bf16) {
    const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(md.G) + idx;
    if (vec) {
      uint2 u = *reinterpret_cast<const uint2*>(src);
      float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.x));
      float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.y));
      g[0] = a.x; g[1] = a.y; g[2] = b.x; g[3] = b.y;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) g[e] = (e < valid) ? __bfloat162float(src[e]) : 0.0f;
    }
  } else {
    const float* src = reinterpret_cast<const float*>(md.G) + idx;
    if (vec) {
      float4 u = *reinterpret_cast<const float4*>(src);
      g[0] = u.x; g[1] = u.y; g[2] = u.z; g[3] = u.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) g[e] = (e < valid) ? src[e] : 0.0f;
    }
  }
}

template <typename E>
__global__ void __launch_bounds__(kPThreads) prologue_kernel(const __grid_constant__ ElemParams p) {
  __shared__ float sM[kPT][kPT + 1];
  __shared__ float red[kPThreads / 32];
  const int tid = threadIdx.x;
  const int ty = tid >> 4;  // 0..15
  const int tx = tid & 15;  // 0..15: 4 consecutive columns each
  for (int64_t t = blockIdx.x; t < p.ntiles; t += gridDim.x) {
    const int mi = find_slot64(p.ptile_prefix, p.nmat, t);
    const MatDesc& md = p.mats[mi];
    const int64_t local = t - __ldg(p.ptile_prefix + mi);
    const int64_t tr = local / md.ptiles_c, tc = local - tr * md.ptiles_c;
    const int64_t r0 = tr * kPT, c0 = tc * kPT;
    const int64_t rows = md.rows, cols = md.cols;
    E* X = reinterpret_cast<E*>(md.X[0]);
    E* Xo = reinterpret_cast<E*>(md.Xop[0]);
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t r = r0 + ty + 16 * i;
      const int64_t c = c0 + tx * 4;
      float M[4] = {0.f, 0.f, 0.f, 0.f};
      if (r < rows && c < cols) {
        const int valid = (cols - c >= 4) ? 4 : static_cast<int>(cols - c);
        const bool vec = md.vec4 && valid == 4;
        const int64_t idx = r * cols + c;
        float g[4];
        load4_in<E>(md, idx, vec, valid, g);
        if (md.buf != nullptr) {
          float* bp = md.buf + idx;
          float b[4];
          if (vec) {
            float4 u = *reinterpret_cast<const float4*>(bp);
            b[0] = u.x; b[1] = u.y; b[2] = u.z; b[3] = u.w;
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) b[e] = (e < valid) ? bp[e] : 0.0f;
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // buf <- fl(fl(mu * buf) + g): two roundings, never fused.
            b[e] = __fadd_rn(__fmul_rn(p.mu, b[e]), g[e]);
            M[e] = p.nesterov ? fmaf(p.mu, b[e], g[e]) : b[e];
          }
          if (vec) {
            *reinterpret_cast<float4*>(bp) = make_float4(b[0], b[1], b[2], b[3]);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (e < valid) bp[e] = b[e];
          }
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) M[e] = g[e];
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (e >= valid) M[e] = 0.0f;
          ss = fmaf(M[e], M[e], ss);
        }
        if (!md.T) {
          E* dst = X + r * md.ldx + c;
          if (valid == 4 && sizeof(E) == 2) {
            __nv_bfloat162 lo = __floats2bfloat162_rn(M[0], M[1]);
            __nv_bfloat162 hi = __floats2bfloat162_rn(M[2], M[3]);
            uint2 u;
            u.x = *reinterpret_cast<uint32_t*>(&lo);
            u.y = *reinterpret_cast<uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(dst) = u;
          } else if (valid == 4) {
            *reinterpret_cast<float4*>(dst) = make_float4(M[0], M[1], M[2], M[3]);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (e < valid) dst[e] = from_f<E>(M[e]);
          }
          if (sizeof(E) == 4 && Xo != X) {
            E* odst = Xo + r * md.ldx + c;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (e < valid) odst[e] = from_f<E>(op_round<E>(M[e]));
          }
        }
      }
      if (md.T) {
#pragma unroll
        for (int e = 0; e < 4; ++e) sM[ty + 16 * i][tx * 4 + e] = M[e];
      }
    }
    if (md.T) {
      __syncthreads();
      // X row = parameter column, X columns = parameter rows.
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int cc = ty + 16 * i;
        const int64_t xr = c0 + cc;
        const int64_t xc = r0 + tx * 4;
        if (xr < cols && xc < rows) {
          E* dst = X + xr * md.ldx + xc;
          const int valid = (rows - xc >= 4) ? 4 : static_cast<int>(rows - xc);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (e < valid) dst[e] = from_f<E>(sM[tx * 4 + e][cc]);
          if (sizeof(E) == 4 && Xo != X) {
            E* odst = Xo + xr * md.ldx + xc;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (e < valid) odst[e] = from_f<E>(op_round<E>(sM[tx * 4 + e][cc]));
          }
        }
      }
      __syncthreads();
    }
    // Fixed-order block reduction of the tile's sum of squares.
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

// One warp per matrix: s = 1 / (sqrt(sum of partials) + 1e-7), summed in a
// fixed order (deterministic).
__global__ void finalize_kernel(const __grid_constant__ ElemParams p) {
  const int mi = blockIdx.x;
  const int lane = threadIdx.x;
  const int64_t b = p.ptile_prefix[mi], e = p.ptile_prefix[mi + 1];
  double acc = 0.0;
  for (int64_t i = b + lane; i < e; i += 32) acc += static_cast<double>(p.partials[i]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) *p.mats[mi].scale = static_cast<float>(1.0 / (sqrt(acc) + 1e-7));
}

// ns_steps == 0: the result is X0 = s M itself.
template <typename E>
__global__ void __launch_bounds__(kPThreads) apply_kernel(const __grid_constant__ ElemParams p) {
  for (int64_t t = blockIdx.x; t < p.ntiles; t += gridDim.x) {
    const int mi = find_slot64(p.ptile_prefix, p.nmat, t);
    const MatDesc& md = p.mats[mi];
    const int64_t local = t - __ldg(p.ptile_prefix + mi);
    const int64_t tr = local / md.ptiles_c, tc = local - tr * md.ptiles_c;
    const float s = *md.scale;
    const float lr = p.lr * md.lr_mult;
    const float decay = 1.0f - lr * p.wd;
    const E* X = reinterpret_cast<const E*>(md.X[0]);
    E* W = reinterpret_cast<E*>(md.W);
    for (int k = threadIdx.x; k < kPT * kPT; k += blockDim.x) {
      const int64_t r = tr * kPT + k / kPT, c = tc * kPT + k % kPT;
      if (r >= md.rows || c >= md.cols) continue;
      const float x = s * to_f<E>(md.T ? X[c * md.ldx + r] : X[r * md.ldx + c]);
      E* wp = W + r * md.cols + c;
      if (md.mode == kModeOrtho) *wp = from_f<E>(x);
      else *wp = from_f<E>(fmaf(to_f<E>(*wp), decay, -lr * x));
    }
  }
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
