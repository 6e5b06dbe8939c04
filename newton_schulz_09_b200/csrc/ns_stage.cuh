// Newton-Schulz stage kernels of the batched Muon update on sm_100a: one
// persistent, warp-specialised tcgen05/TMEM/TMA launch per stage for every
// matrix of a group.  ns_stage_kernel runs the GEMM X' = c (a X + (A or P) X)
// with the fused combine or weight update, and the quintic SQUARE
// P = b A + c A A, and the SYRK with 128 x 256 tiles for groups too small to
// fill the SMs with the 256 x 256 tiles of syrk256_kernel (syrk256.cuh).
//
// Sources: DMuon blog post "DMuon：让矩阵正交化优化器达到接近 AdamW 的分布式训练开销",
// section "Muon 核心：Newton-Schulz 迭代" (the cubic step and the transpose
// rule); DMuon training guide "训练指南", section "超参数指南" (custom
// coefficients).  Included by kernels.cuh, which defines the descriptors.
#pragma once

namespace dmuon {
// Upper-triangle SYRK tiles of one matrix, enumerated column-band major:
// column band J (256 wide) holds row bands I = 0 .. 2J+1 (128 tall), so band
// J starts at J (J + 1).  The last tile of a band, I = 2J+1, lies on the
// diagonal with its left 128 columns wholly below it: that tile is computed
// as a 128 x 128 half tile (UMMA N = 128) over the band's right 128 columns.
__device__ __forceinline__ void syrk_tile_coords(int local, int& I, int& J) {
  int j = static_cast<int>((sqrtf(4.0f * static_cast<float>(local) + 1.0f) - 1.0f) * 0.5f);
  while ((j + 1) * (j + 2) <= local) ++j;
  while (j * (j + 1) > local) --j;
  J = j;
  I = local - j * (j + 1);
}

struct TileInfo {
  int mi, tm, tn, nkb;
  int half;   // SYRK: 128 x 128 tile over columns tn * 256 + 128 ..
};

// Tile t of a launch (128 x 256 tiles).  kPair: the GEMM's tiles are
// 256 x 256 pairs, and CTA `rank` of the pair takes rows 128 rank .. of it.
template <int kMode, int BK, bool kPair = false>
__device__ __forceinline__ TileInfo decode_tile(const NsParams& p, int t, int rank = 0) {
  TileInfo ti;
  const int slot = find_slot(p.tile_prefix, p.nmat, t);
  ti.mi = __ldg(p.order + slot);
  const int local = t - __ldg(p.tile_prefix + slot);
  const MatDesc& md = p.mats[ti.mi];
  ti.half = 0;
  if (kMode == kSyrk || kMode == kSquare) {
    syrk_tile_coords(local, ti.tm, ti.tn);
    ti.nkb = ((kMode == kSyrk ? md.n : md.m) + BK - 1) / BK;
    ti.half = (ti.tm == 2 * ti.tn + 1) ? 1 : 0;
  } else if (kPair) {
    const int nI = (md.m + 2 * kBM - 1) / (2 * kBM);
    ti.tn = local / nI;
    ti.tm = 2 * (local - ti.tn * nI) + rank;
    ti.nkb = (md.m + BK - 1) / BK;
  } else {
    const int nI = (md.m + kBM - 1) / kBM;
    ti.tn = local / nI;
    ti.tm = local - ti.tn * nI;
    ti.nkb = (md.m + BK - 1) / BK;
  }
  return ti;
}

// ======================================================================
// Epilogue (warps 2-5): TMEM accumulators of this CTA's 128 tile rows ->
// SYRK stores (A and its mirror), or the GEMM combine / final update.
// The accumulator buffer is released by `release(b)` once fully read.
// Returns false when a bounded wait gave up.
// ======================================================================
// The epilogue's waits: sleeping in try_wait on one CTA, polling in the pair
// kernel (whose accumulators arrive by a commit from the other SM).
template <bool kPair>
__device__ __forceinline__ bool epi_wait(uint64_t* bar, uint32_t parity, const NsParams& p) {
  return kPair ? mbar_wait_spin(bar, parity, p.err, p.wait_limit_ns)
               : mbar_wait(bar, parity, p.err, p.wait_limit_ns);
}

template <int kMode, typename E, bool kPair = false, typename Release>
__device__ __forceinline__ bool run_epilogue(const NsParams& p, uint32_t tmem_base, uint8_t* epi,
                                             uint64_t* tfull, uint64_t* xfull, int warp, int lane,
                                             int t0, int tstride, Release release, int rank = 0) {
  constexpr int EB = static_cast<int>(sizeof(E));
  constexpr int BK = 128 / EB;
  const int q4 = warp & 3;                 // TMEM lane quarter of this warp
  const int row_in_tile = q4 * 32 + lane;
  bool ok = true;

  if (kMode == kGemm && EB == 2 && !p.last) {
    // bf16 GEMM steps: the old X arrives by TMA, 64 columns (one quarter) at
    // a time, into a two-slot ring; each thread combines its row in place
    // with the accumulator and the quarter leaves by TMA store.
    const bool leader = (warp == 2 && lane == 0);
    int ld_t = t0, ld_q = 0;               // next quarter to load (leader only)
    uint32_t ld_g = 0;
    int fenced = -1;                       // matrix whose maps the leader has acquired
    bool slot_busy[kEpiSlots] = {false, false};
    uint32_t slot_phase[kEpiSlots] = {0u, 0u};
    auto quarters_of = [&](const TileInfo& ti) -> int {
      const int left = p.mats[ti.mi].n - ti.tn * kBN;
      const int nq = (left + 63) / 64;
      return nq < 4 ? nq : 4;
    };
    auto load_next = [&]() {
      if (ld_t >= p.ntiles) return;
      const TileInfo ti = decode_tile<kMode, BK, kPair>(p, ld_t, rank);
      if (ti.mi != fenced) {
        tensormap_acquire_gpu(&p.maps[ti.mi].xk[p.cur]);
        tensormap_acquire_gpu(&p.maps[ti.mi].xk[p.cur ^ 1]);
        fenced = ti.mi;
      }
      const int slot = static_cast<int>(ld_g & 1u);
      mbar_arrive_expect_tx(&xfull[slot], kEpiSlotBytes);
      tma_load_2d(epi + slot * kEpiSlotBytes, &p.maps[ti.mi].xk[p.cur], &xfull[slot],
                  ti.tn * kBN + 64 * ld_q, ti.tm * kBM);
      slot_busy[slot] = true;
      slot_phase[slot] = (ld_g >> 1) & 1u;
      ++ld_g;
      if (++ld_q >= quarters_of(ti)) { ld_q = 0; ld_t += tstride; }
    };
    if (leader) { load_next(); load_next(); }
    uint32_t g = 0;
    int lt = 0;
    for (int t = t0; t < p.ntiles && ok; t += tstride, ++lt) {
      const TileInfo ti = decode_tile<kMode, BK, kPair>(p, t, rank);
      const MatDesc& md = p.mats[ti.mi];
      const int b = lt & 1;
      const uint32_t tph = (static_cast<uint32_t>(lt) >> 1) & 1u;
      const float cs = p.first ? *md.scale : 1.0f;
      const int nq = quarters_of(ti);
      bool w = epi_wait<kPair>(&tfull[b], tph, p);
      if (!named_bar_and(1, 128, w)) { ok = false; break; }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q4 * 32) << 16) + static_cast<uint32_t>(b * kBN);
      for (int qq = 0; qq < nq; ++qq, ++g) {
        const int slot = static_cast<int>(g & 1u);
        w = epi_wait<kPair>(&xfull[slot], (g >> 1) & 1u, p);
        if (!named_bar_and(1, 128, w)) { ok = false; break; }
        uint32_t v0[32], v1[32];
        tmem_ld32(taddr + qq * 64, v0);
        tmem_ld32(taddr + qq * 64 + 32, v1);
        tmem_ld_wait();
        if (qq == nq - 1) release(b);
        uint8_t* rowp = epi + slot * kEpiSlotBytes + row_in_tile * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4* ptr = reinterpret_cast<uint4*>(rowp + ((c ^ (row_in_tile & 7)) << 4));
          uint4 u = *ptr;
          uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 xf = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&wv[j]));
            const int col = c * 8 + 2 * j;
            const float a0 = __uint_as_float(col < 32 ? v0[col] : v1[col - 32]);
            const float a1 = __uint_as_float(col + 1 < 32 ? v0[col + 1] : v1[col + 1 - 32]);
            __nv_bfloat162 yv = __floats2bfloat162_rn(cs * (p.ca * xf.x + p.cb * a0),
                                                      cs * (p.ca * xf.y + p.cb * a1));
            wv[j] = *reinterpret_cast<uint32_t*>(&yv);
          }
          *ptr = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (leader) {
          // (the odd CTA of a pair tile that ends inside the matrix's last
          // 128 rows holds no rows of it: nothing to store)
          if (ti.tm * kBM < md.m)
            tma_store_2d(&p.maps[ti.mi].xk[p.cur ^ 1], epi + slot * kEpiSlotBytes,
                         ti.tn * kBN + 64 * qq, ti.tm * kBM);
          bulk_commit_group();
          bulk_wait_group_read0();               // slot read out: it may be refilled
          slot_busy[slot] = false;
          load_next();
        }
      }
    }
    if (leader) {
      bulk_wait_group0();
      if (!ok)
        for (int e = 0; e < kEpiSlots; ++e)
          if (slot_busy[e]) mbar_wait(&xfull[e], slot_phase[e], nullptr, p.wait_limit_ns, 1024);
    }
    return ok;
  }

  int lt = 0;
  for (int t = t0; t < p.ntiles && ok; t += tstride, ++lt) {
    const TileInfo ti = decode_tile<kMode, BK, kPair>(p, t, rank);
    const MatDesc& md = p.mats[ti.mi];
    const int b = lt & 1;
    const uint32_t tph = (static_cast<uint32_t>(lt) >> 1) & 1u;
    const float s = *md.scale;
    bool w = epi_wait<kPair>(&tfull[b], tph, p);
    if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
    tc_fence_after();
    const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q4 * 32) << 16) + static_cast<uint32_t>(b * kBN);
    const int R = ti.tm * kBM + row_in_tile;
    const int m = md.m, n = md.n;
    if (kMode == kSyrk || kMode == kSquare) {
      // SYRK: A = s^2 X X^T on the first step.  SQUARE: P = cb A + cc A A,
      // A read back in the tile's own rows and columns.
      const float alpha = (kMode == kSquare) ? p.cc : (p.first ? s * s : 1.0f);
      E* A = reinterpret_cast<E*>(kMode == kSquare ? md.P : md.A);
      const E* Asrc = reinterpret_cast<const E*>(md.A);
      const int64_t lda = md.lda;
      const int nch = ti.half ? kBN / 64 : kBN / 32;
      const int col0 = ti.tn * kBN + (ti.half ? kBN / 2 : 0);
#pragma unroll 1
      for (int c = 0; c < nch; ++c) {
        uint32_t v[32];
        tmem_ld32(taddr + c * 32, v);
        tmem_ld_wait();
        if (c == nch - 1) release(b);
        const int C0 = col0 + c * 32;
        if (R < m && C0 < m && (!p.mirror || C0 + 31 >= R)) {
          float y[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) y[j] = alpha * __uint_as_float(v[j]);
          if (kMode == kSquare) {
            float a0[32];
            const E* srow = Asrc + static_cast<int64_t>(R) * lda + C0;
            if (C0 + 32 <= m) {
              load32<E>(srow, a0);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) a0[j] = (C0 + j < m) ? to_f<E>(srow[j]) : 0.0f;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) y[j] = fmaf(p.cb, a0[j], y[j]);
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) y[j] = op_round<E>(y[j]);
          E* arow = A + static_cast<int64_t>(R) * lda;
          if (!p.mirror) {
            // Upper tiles and whole diagonal 128-blocks: every computed element
            // is stored once, nothing is mirrored (the GEMM reads the lower
            // part transposed).
            if (C0 + 32 <= m) {
              store32<E>(arow + C0, y);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (C0 + j < m) arow[C0 + j] = from_f<E>(y[j]);
            }
            if (p.diag_full && !ti.half && ti.tm == 2 * ti.tn && C0 >= col0 + kBN / 2) {
              // the diagonal 256-block's upper-right quarter, mirrored into its
              // lower-left one (lanes are consecutive R: contiguous runs)
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (C0 + j < m) A[static_cast<int64_t>(C0 + j) * lda + R] = from_f<E>(y[j]);
            }
            continue;
          }
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
        if (c == kBN / 32 - 1) release(b);
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
          for (int j = 0; j < 32; ++j) y[j] = cs * (p.ca * x[j] + p.cb * __uint_as_float(v[j]));
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
            // consecutive R, so each j touches one contiguous run.  All
            // loads are issued before any store so they overlap.
            E* wcol = W + static_cast<int64_t>(C0) * cols + R;
            if (md.mode == kModeOrtho) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (C0 + j < n) wcol[static_cast<int64_t>(j) * cols] = from_f<E>(y[j]);
            } else {
              float wv[32];
#pragma unroll
              for (int j = 0; j < 32; ++j)
                wv[j] = (C0 + j < n) ? to_f<E>(wcol[static_cast<int64_t>(j) * cols]) : 0.0f;
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (C0 + j < n)
                  wcol[static_cast<int64_t>(j) * cols] = from_f<E>(fmaf(wv[j], decay, -lr * y[j]));
            }
          }
        }
      }
    }
  }
  return ok;
}

// ======================================================================
// Newton-Schulz stage kernel, one CTA per 128 x 256 tile.
// Persistent and warp specialised: warp 0 TMA producer, warp 1 UMMA issuer,
// warps 2-5 epilogue.
// ======================================================================
template <int kMode, typename E>
__global__ void __launch_bounds__(kNsThreads, 1) ns_stage_kernel(const __grid_constant__ NsParams p) {
  constexpr int EB = static_cast<int>(sizeof(E));
  constexpr int BK = 128 / EB;              // K elements per stage (one 128-byte row)
  constexpr int MMA_K = 32 / EB;            // K per UMMA instruction
  constexpr int KSTEPS = BK / MMA_K;        // = 4
  constexpr uint32_t FMT = (EB == 2) ? 1u : 2u;
  constexpr uint32_t IDESC = make_idesc(FMT, 0u, kMode == kGemm ? 1u : 0u, kBM, kBN);
  constexpr uint32_t IDESC_HALF = make_idesc(FMT, 0u, 0u, kBM, kBN / 2);   // SYRK / SQUARE half tiles
  constexpr uint32_t IDESC_AT = make_idesc(FMT, 1u, 1u, kBM, kBN);         // GEMM, A k-block MN-major
  // SQUARE from an upper-only A: k-blocks with both operands MN-major, or only B
  constexpr uint32_t IDESC_TT_HALF = make_idesc(FMT, 1u, 1u, kBM, kBN / 2);
  constexpr uint32_t IDESC_KT = make_idesc(FMT, 0u, 1u, kBM, kBN);
  constexpr uint32_t IDESC_KT_HALF = make_idesc(FMT, 0u, 1u, kBM, kBN / 2);
  constexpr int NBOX_B = (kMode == kGemm) ? kBN / BK : 2;
  constexpr uint32_t BOX_B_BYTES = (kMode == kGemm) ? BK * 128 : kAStageBytes;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sa = smem;
  uint8_t* sb = smem + kStages * kAStageBytes;
  uint8_t* epi = sb + kStages * kBStageBytes;          // GEMM output quarters (bf16)
  uint64_t* full = reinterpret_cast<uint64_t*>(epi + kEpiSlots * kEpiSlotBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* xfull = tempty + 2;                          // [kEpiSlots]
  uint64_t* drain = xfull + kEpiSlots;
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
    for (int e = 0; e < kEpiSlots; ++e) mbar_init(&xfull[e], 1);
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
  // Barriers and TMEM were set up without touching global memory, while the
  // previous kernel in the stream may still run (no CTA of another stage
  // kernel fits beside this one's shared memory, so the TMEM is free); from
  // here on its results are needed.
  griddep_wait();
  griddep_launch_dependents();

  bool ok = true;
  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_phase[kStages];
    bool issued[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) { issued[s] = false; issued_phase[s] = 0; }
    int fenced = -1;     // matrix whose tensor maps this thread has acquired
    for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x) {
      const TileInfo ti = decode_tile<kMode, BK>(p, t);
      const MatDesc& md = p.mats[ti.mi];
      const MatMaps& mp = p.maps[ti.mi];
      // SYRK: X X^T (both operands X, K-major).  SQUARE: A A (both operands A,
      // K-major; A is symmetric, so A A = A A^T).  GEMM: A (or P) times X (MN-major).
      const CUtensorMap* mapA = (kMode == kSyrk) ? &mp.xk[p.cur]
                              : (kMode == kSquare) ? &mp.a : (p.quintic ? &mp.p : &mp.a);
      const CUtensorMap* mapB = (kMode == kSyrk) ? &mp.xk[p.cur]
                              : (kMode == kSquare) ? &mp.a : &mp.xmn[p.cur];
      const CUtensorMap* mapBw = (kMode == kSyrk) ? &mp.xkw[p.cur] : &mp.aw;
      const CUtensorMap* mapAt = (kMode == kGemm && p.quintic) ? &mp.pmn : &mp.amn;
      // k-blocks read from the upper triangle, A[k rows][M columns], MN-major:
      // the GEMM's A operand left of the row block's diagonal 128-block; with
      // a_upper in the SQUARE stage (A holds its upper triangle and whole
      // diagonal 256-blocks), the A operand left of its row block's diagonal
      // 256-block and the B operand left of the tile's column band.
      const int kb_t = !p.a_upper ? 0
                     : (kMode == kGemm) ? ti.tm * (kBM / BK)
                     : (kMode == kSquare) ? (ti.tm >> 1) * (2 * kBM / BK) : 0;
      const int kb_bt = (kMode == kSquare && p.a_upper) ? ti.tn * (kBN / BK) : 0;
      int nb = 0;
      const int b_row0 = ti.tn * kBN + (ti.half ? kBN / 2 : 0);   // SYRK / SQUARE B operand rows
      if (kMode == kSyrk || kMode == kSquare) {
        nb = (ti.half || ti.tn * kBN + 128 >= md.m) ? 1 : 2;
      } else if (md.b3d) {
        nb = NBOX_B;   // the 3-D box is always whole: blocks past the last column arrive as zeros
      } else {
        const int left = md.n - ti.tn * kBN;
        nb = (left + BK - 1) / BK;
        if (nb > NBOX_B) nb = NBOX_B;
      }
      // Diagonal tiles of the SYRK / SQUARE: on the full one (I = 2J) the A
      // operand's 128 rows are the first half of the B operand's 256, on the
      // half tile (I = 2J+1) the B rows are the A rows.  One load serves both.
      const bool a_in_b = (kMode != kGemm) && !ti.half && ti.tm == 2 * ti.tn;
      const bool b_is_a = (kMode != kGemm) && ti.half;
      const uint32_t bytes = (a_in_b ? 0u : static_cast<uint32_t>(kAStageBytes)) +
                             (b_is_a ? 0u : static_cast<uint32_t>(nb) * BOX_B_BYTES);
      if (lane == 0 && ti.mi != fenced) {
        // The maps were written by a kernel (plan upload): order that write
        // before TMA reads them.
        tensormap_acquire_gpu(mapA);
        tensormap_acquire_gpu(mapB);
        if (kMode != kGemm) tensormap_acquire_gpu(mapBw);
        if ((kMode == kGemm || kMode == kSquare) && p.a_upper) {
          tensormap_acquire_gpu(mapAt);
          if (kMode == kSquare && md.a3d) {
            tensormap_acquire_gpu(&mp.amn3[0]);
            tensormap_acquire_gpu(&mp.amn3[1]);
          }
        }
        fenced = ti.mi;
      }
      for (int kb = 0; kb < ti.nkb; ++kb) {
        bool w = mbar_wait_spin(&empty[stage], phase ^ 1u, p.err, p.wait_limit_ns);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[stage], bytes);
          uint8_t* a_dst = sa + stage * kAStageBytes;
          uint8_t* b_dst = sb + stage * kBStageBytes;
          if (kb < kb_t && !a_in_b) {
            // 128 M columns in 128-byte chunks (2 for bf16, 4 for fp32), each
            // BK rows of K: the MN-major layout of the B operand.  The SQUARE
            // stage loads both 64-column blocks at once through A's 3-D view
            // (for the GEMM's A operand one load measured slower than two).
            if (kMode == kSquare && EB == 2 && md.a3d) {
              tma_load_3d(a_dst, &mp.amn3[1], &full[stage], 0, kb * BK, ti.tm * (kBM / 64));
            } else {
#pragma unroll
              for (int h = 0; h < EB; ++h)
                tma_load_2d(a_dst + h * (BK * 128), mapAt, &full[stage], ti.tm * kBM + h * (128 / EB), kb * BK);
            }
          } else if (!a_in_b) {
            tma_load_2d(a_dst, mapA, &full[stage], kb * BK, ti.tm * kBM);
          }
          if (kMode == kGemm && md.b3d) {
            // The four 64-column blocks of the tile in one load, same smem layout.
            tma_load_3d(b_dst, mapB, &full[stage], 0, kb * BK, ti.tn * (kBN / 64));
          } else if (b_is_a) {
            // half tile: its B rows are its A rows, already loaded
          } else if (kMode == kSquare && kb < kb_bt) {
            // the B operand's rows as columns of the upper triangle, in
            // 128-byte chunks of BK rows of K (MN-major, as the GEMM's X):
            // one 3-D load of nb x 2 column blocks, else one 2-D box per chunk
            if (EB == 2 && md.a3d) {
              tma_load_3d(b_dst, &mp.amn3[nb == 2 ? 0 : 1], &full[stage], 0, kb * BK, b_row0 / 64);
            } else {
              for (int j = 0; j < nb * EB; ++j)
                tma_load_2d(b_dst + j * (BK * 128), mapAt, &full[stage], b_row0 + j * (128 / EB), kb * BK);
            }
          } else if (kMode != kGemm && nb == 2) {
            // Both 128-row halves of the B operand in one 256-row load.
            tma_load_2d(b_dst, mapBw, &full[stage], kb * BK, b_row0);
          } else {
            for (int j = 0; j < nb; ++j) {
              if (kMode != kGemm)
                tma_load_2d(b_dst + j * kAStageBytes, mapB, &full[stage], kb * BK, b_row0 + j * 128);
              else
                tma_load_2d(b_dst + j * BOX_B_BYTES, mapB, &full[stage], ti.tn * kBN + j * BK, kb * BK);
            }
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
      bool w = mbar_wait_spin(&tempty[b], tph ^ 1u, p.err, p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * kBN);
      const uint32_t idesc = (kMode != kGemm && ti.half) ? IDESC_HALF : IDESC;
      const int kb_t = !p.a_upper ? 0                                            // as the producer
                     : (kMode == kGemm) ? ti.tm * (kBM / BK)
                     : (kMode == kSquare) ? (ti.tm >> 1) * (2 * kBM / BK) : 0;
      const int kb_bt = (kMode == kSquare && p.a_upper) ? ti.tn * (kBN / BK) : 0;
      const bool a_in_b = (kMode != kGemm) && !ti.half && ti.tm == 2 * ti.tn;   // as the producer
      const bool b_is_a = (kMode != kGemm) && ti.half;
      for (int kb = 0; kb < ti.nkb; ++kb) {
        w = mbar_wait_spin(&full[stage], phase, p.err, p.wait_limit_ns);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_own = smem_u32(sa + stage * kAStageBytes);
          const uint32_t b_own = smem_u32(sb + stage * kBStageBytes);
          const uint32_t a_base = a_in_b ? b_own : a_own;
          const uint32_t b_base = b_is_a ? a_own : b_own;
          const bool at = kb < kb_t;      // A k-block transposed (MN-major)
          const bool bt = kMode == kGemm || kb < kb_bt;   // B operand MN-major
#pragma unroll
          for (int k = 0; k < KSTEPS; ++k) {
            const uint64_t ad =
                at ? sw128_desc(a_base + k * MMA_K * 128, BK * 128, EB == 2 ? 1024 : 512,
                                EB == 2 ? kSwizzle128B : kSwizzle128B32)
                   : sw128_desc(a_base + k * 32, 16, 1024);
            // MN-major B: 16-bit operands use the 16-byte-unit swizzle (8-line
            // K groups); 32-bit operands must use 32-byte units (4-line groups).
            const uint64_t bd =
                !bt ? sw128_desc(b_base + k * 32, 16, 1024)
                    : sw128_desc(b_base + k * MMA_K * 128, BK * 128, EB == 2 ? 1024 : 512,
                                 EB == 2 ? kSwizzle128B : kSwizzle128B32);
            const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
            const uint32_t id = (kMode == kSquare)
                                    ? (at ? (ti.half ? IDESC_TT_HALF : IDESC_AT)
                                          : bt ? (ti.half ? IDESC_KT_HALF : IDESC_KT) : idesc)
                                    : (at ? IDESC_AT : idesc);
            if (EB == 2) umma_f16(d_tmem, ad, bd, id, acc);
            else umma_tf32(d_tmem, ad, bd, id, acc);
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
    ok = run_epilogue<kMode, E>(p, tmem_base, epi, tfull, xfull, warp, lane, blockIdx.x, gridDim.x,
                                [&](int b) {
                                         tc_fence_before();
                                         mbar_arrive(&tempty[b]);
                                       });
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}


}  // namespace dmuon
