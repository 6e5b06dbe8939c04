// SYRK stage of the batched Muon update on sm_100a: A = X X^T over upper
// 256 x 256 tiles, one persistent warp-specialised tcgen05/TMEM/TMA launch for
// every matrix of a group.
//
// Source: DMuon blog post "DMuon：让矩阵正交化优化器达到接近 AdamW 的分布式训练开销",
// section "Muon 核心：Newton-Schulz 迭代" (A = G G^T of the cubic step).
// Included by kernels.cuh after ns_stage.cuh (shared helpers and descriptors).
#pragma once

namespace dmuon {
// ======================================================================
// SYRK with 256 x 256 tiles per CTA.  A is stored as its upper triangle and
// diagonal 128-blocks (with diag_full: diagonal 256-blocks, for the pair
// GEMM), or in full (mirrored) when a quintic SQUARE stage on 128 x 256 tiles
// reads it K-major.  Each k-block brings 256 rows of X for the A operand
// and 256 for the B operand (64 KB) and feeds two 128 x 256 UMMA halves that
// share the B operand: a third fewer operand bytes per FLOP than 128 x 256
// tiles.  The two fp32 accumulators take all 512 TMEM columns, so a tile's
// epilogue is not overlapped with the next tile's MMAs; with K = n in the
// thousands that costs a few percent of the stage.  Diagonal tiles (I = J)
// load one box for both operands, and their second half is 128 x 128 (the
// block's lower-left quarter is below the diagonal).
// Same warp roles as ns_stage_kernel; three 64 KB pipeline stages.
// ======================================================================
constexpr int kS2Stages = 3;
constexpr int kS2OpBytes = kBN * 128;              // 256 rows x 128 bytes of K
// + two 16 KB slots (128 rows x 64 bf16 columns) through which the epilogue
// stages its stores for TMA
constexpr int kS2SmemBytes = kS2Stages * 2 * kS2OpBytes + kEpiSlots * kEpiSlotBytes + 1024 /*align*/ + 256;
static_assert(kS2SmemBytes <= 232448, "exceeds the 227 KB of shared memory per block");

// Upper-triangle 256 x 256 tiles of one matrix, column-band major: band J
// holds I = 0 .. J and starts at J (J + 1) / 2.
__device__ __forceinline__ void syrk256_tile_coords(int local, int& I, int& J) {
  int j = static_cast<int>((sqrtf(8.0f * static_cast<float>(local) + 1.0f) - 1.0f) * 0.5f);
  while ((j + 1) * (j + 2) / 2 <= local) ++j;
  while (j * (j + 1) / 2 > local) --j;
  J = j;
  I = local - j * (j + 1) / 2;
}

struct Tile256 {
  int mi, I, J, nkb;
  bool diag;
};

template <int BK, int kMode = kSyrk>
__device__ __forceinline__ Tile256 decode_tile256(const NsParams& p, int t) {
  Tile256 ti;
  const int slot = find_slot(p.tile_prefix, p.nmat, t);
  ti.mi = __ldg(p.order + slot);
  syrk256_tile_coords(t - __ldg(p.tile_prefix + slot), ti.I, ti.J);
  ti.nkb = ((kMode == kSquare ? p.mats[ti.mi].m : p.mats[ti.mi].n) + BK - 1) / BK;
  ti.diag = ti.I == ti.J;
  return ti;
}

// kMode == kSquare: the quintic SQUARE stage P = cb A + cc A A on the same
// tiles (bf16 groups on CTA pairs only).  Its operands are rows of A, K = m;
// A holds its upper triangle and whole diagonal 256-blocks, so an operand's
// k-blocks left of its own diagonal 256-block come transposed from the upper
// triangle (one 3-D load through A's MN-major view, MN-major descriptors).
// The epilogue adds cb A, read back from A's tile, and stores P like A.
template <typename E, int kMode = kSyrk>
__global__ void __launch_bounds__(kNsThreads, 1) syrk256_kernel(const __grid_constant__ NsParams p) {
  constexpr int EB = static_cast<int>(sizeof(E));
  constexpr int BK = 128 / EB;
  constexpr int MMA_K = 32 / EB;
  constexpr int KSTEPS = BK / MMA_K;
  constexpr uint32_t FMT = (EB == 2) ? 1u : 2u;
  constexpr uint32_t IDESC = make_idesc(FMT, 0u, 0u, kBM, kBN);
  constexpr uint32_t IDESC_HALF = make_idesc(FMT, 0u, 0u, kBM, kBN / 2);
  // SQUARE k-blocks with the B operand, or both operands, MN-major
  constexpr uint32_t IDESC_KT = make_idesc(FMT, 0u, 1u, kBM, kBN);
  constexpr uint32_t IDESC_KT_HALF = make_idesc(FMT, 0u, 1u, kBM, kBN / 2);
  constexpr uint32_t IDESC_TT = make_idesc(FMT, 1u, 1u, kBM, kBN);
  constexpr uint32_t IDESC_TT_HALF = make_idesc(FMT, 1u, 1u, kBM, kBN / 2);
  static_assert(kMode == kSyrk || EB == 2, "the SQUARE mode is bf16 only");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  // stage s: A operand rows at s * 64 KB, B operand rows 32 KB after them
  uint8_t* epi = smem + kS2Stages * 2 * kS2OpBytes;    // bf16 store slots
  uint64_t* full = reinterpret_cast<uint64_t*>(epi + kEpiSlots * kEpiSlotBytes);
  uint64_t* empty = full + kS2Stages;
  uint64_t* tfull = empty + kS2Stages;
  uint64_t* tempty = tfull + 1;
  uint64_t* drain = tempty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kS2Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 4 * 32);
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
    uint32_t issued_phase[kS2Stages];
    bool issued[kS2Stages];
#pragma unroll
    for (int s = 0; s < kS2Stages; ++s) { issued[s] = false; issued_phase[s] = 0; }
    int fenced = -1;
    for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x) {
      const Tile256 ti = decode_tile256<BK, kMode>(p, t);
      const MatMaps& mp = p.maps[ti.mi];
      // 256-row K-major boxes of X (SYRK) or A (SQUARE)
      const CUtensorMap* map = (kMode == kSquare) ? &mp.aw : &mp.xkw[p.cur];
      // SQUARE: k-blocks left of the A rows' (B rows') diagonal 256-block
      const int kb_at = (kMode == kSquare) ? ti.I * (kBN / BK) : 0;
      const int kb_bt = (kMode == kSquare) ? ti.J * (kBN / BK) : 0;
      if (lane == 0 && ti.mi != fenced) {
        tensormap_acquire_gpu(map);
        if (kMode == kSquare) tensormap_acquire_gpu(&mp.amn3[0]);
        fenced = ti.mi;
      }
      const uint32_t bytes = ti.diag ? kS2OpBytes : 2 * kS2OpBytes;
      for (int kb = 0; kb < ti.nkb; ++kb) {
        bool w = mbar_wait(&empty[stage], phase ^ 1u, p.err, p.wait_limit_ns);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[stage], bytes);
          uint8_t* a_dst = smem + stage * 2 * kS2OpBytes;
          if (!ti.diag) {
            if (kb < kb_at) tma_load_3d(a_dst, &mp.amn3[0], &full[stage], 0, kb * BK, ti.I * (kBN / 64));
            else tma_load_2d(a_dst, map, &full[stage], kb * BK, ti.I * kBN);
          }
          if (kb < kb_bt) tma_load_3d(a_dst + kS2OpBytes, &mp.amn3[0], &full[stage], 0, kb * BK, ti.J * (kBN / 64));
          else tma_load_2d(a_dst + kS2OpBytes, map, &full[stage], kb * BK, ti.J * kBN);
        }
        __syncwarp();
        issued[stage] = true;
        issued_phase[stage] = phase;
        if (++stage == kS2Stages) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok && lane == 0) {
      for (int s = 0; s < kS2Stages; ++s)
        if (issued[s]) mbar_wait(&full[s], issued_phase[s], nullptr, p.wait_limit_ns, 1024);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ UMMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int lt = 0;
    for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x, ++lt) {
      const Tile256 ti = decode_tile256<BK, kMode>(p, t);
      const int kb_at = (kMode == kSquare) ? ti.I * (kBN / BK) : 0;   // as the producer
      const int kb_bt = (kMode == kSquare) ? ti.J * (kBN / BK) : 0;
      bool w = mbar_wait(tempty, (static_cast<uint32_t>(lt) & 1u) ^ 1u, p.err, p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      for (int kb = 0; kb < ti.nkb; ++kb) {
        w = mbar_wait(&full[stage], phase, p.err, p.wait_limit_ns);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t own = smem_u32(smem + stage * 2 * kS2OpBytes);
          const uint32_t b_base = own + kS2OpBytes;
          const uint32_t a_base = ti.diag ? b_base : own;
          const bool at = kb < kb_at, bt = kb < kb_bt;    // MN-major operands (SQUARE)
#pragma unroll
          for (int k = 0; k < KSTEPS; ++k) {
            const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              // a half is 128 rows: 16 KB K-major, or two 8 KB column blocks MN-major
              const uint32_t a_h = a_base + h * (kS2OpBytes / 2);
              const uint64_t ad = at ? sw128_desc(a_h + k * MMA_K * 128, BK * 128, 1024, kSwizzle128B)
                                     : sw128_desc(a_h + k * 32, 16, 1024);
              const bool quarter = ti.diag && h == 1;   // 128 x 128 over the B rows 128 .. 255
              const uint32_t b_q = b_base + (quarter ? kS2OpBytes / 2 : 0);
              const uint64_t bd = bt ? sw128_desc(b_q + k * MMA_K * 128, BK * 128, 1024, kSwizzle128B)
                                     : sw128_desc(b_q + k * 32, 16, 1024);
              const uint32_t id = at ? (quarter ? IDESC_TT_HALF : IDESC_TT)
                                : bt ? (quarter ? IDESC_KT_HALF : IDESC_KT)
                                     : (quarter ? IDESC_HALF : IDESC);
              const uint32_t d = tmem_base + static_cast<uint32_t>(h * kBN);
              if (EB == 2) umma_f16(d, ad, bd, id, acc);
              else umma_tf32(d, ad, bd, id, acc);
            }
          }
          umma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == kS2Stages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(tfull);
      __syncwarp();
    }
    if (!ok && lane == 0) {
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.wait_limit_ns, 1024);
    }
  } else {
    // ------------------------------------------------ epilogue (4 warps)
    const int q4 = warp & 3;
    const int row_in_tile = q4 * 32 + lane;
    int fenced_a = -1;        // matrix whose A map the store leader has acquired
    uint32_t gq = 0;          // store quarters so far (slot ring position)
    int lt = 0;
    for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x, ++lt) {
      const Tile256 ti = decode_tile256<BK, kMode>(p, t);
      const MatDesc& md = p.mats[ti.mi];
      const float s = *md.scale;
      bool w = mbar_wait(tfull, static_cast<uint32_t>(lt) & 1u, p.err, p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      // SYRK: A = alpha X X^T.  SQUARE: P = cc (A A) + cb A.
      const float alpha = (kMode == kSquare) ? p.cc : (p.first ? s * s : 1.0f);
      E* A = reinterpret_cast<E*>(kMode == kSquare ? md.P : md.A);    // the stored matrix
      const E* Asrc = reinterpret_cast<const E*>(md.A);
      const int64_t lda = md.lda;
      const int m = md.m;
      if (EB == 2 && (!p.mirror || kMode == kSquare)) {
        // Upper triangle and diagonal 128-blocks through shared memory: each
        // 128 x 64 quarter goes TMEM -> registers -> a 128B-swizzled slot ->
        // one TMA store into A (clipped at m).  Two slots alternate; a slot
        // is rewritten only after the store two quarters back has read it.
        // The accumulators are released after the tile's last TMEM load.
        const bool leader = (warp == 2 && lane == 0);
        const CUtensorMap* smap = (kMode == kSquare) ? &p.maps[ti.mi].p : &p.maps[ti.mi].a;
        if (leader && ti.mi != fenced_a) {
          tensormap_acquire_gpu(smap);
          fenced_a = ti.mi;
        }
        const int nq0 = kBN / 64;
        const int nq = nq0 + (ti.diag ? kBN / 128 : kBN / 64);
#pragma unroll 1
        for (int qi = 0; qi < nq; ++qi, ++gq) {
          const int h = qi < nq0 ? 0 : 1;
          const int q = qi - h * nq0;
          const bool quarter = ti.diag && h == 1;
          const int R0 = ti.I * kBN + h * kBM;
          const int C0 = ti.J * kBN + (quarter ? kBN / 2 : 0) + q * 64;
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q4 * 32) << 16) +
                                 static_cast<uint32_t>(h * kBN + q * 64);
          // SQUARE: this row's 64 values of A under the quarter (cb A), loaded
          // before the TMEM reads so that both latencies overlap
          uint32_t ar[32];
          if (kMode == kSquare) {
            const int R = R0 + row_in_tile;
            const E* arow = Asrc + static_cast<int64_t>(R) * lda + C0;
            if (R < m && C0 + 64 <= m) {
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const uint4 u = reinterpret_cast<const uint4*>(arow)[i];
                ar[4 * i] = u.x; ar[4 * i + 1] = u.y; ar[4 * i + 2] = u.z; ar[4 * i + 3] = u.w;
              }
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const bool in0 = R < m && C0 + 2 * i < m, in1 = R < m && C0 + 2 * i + 1 < m;
                const __nv_bfloat162 pr = __floats2bfloat162_rn(in0 ? to_f<E>(arow[2 * i]) : 0.0f,
                                                                in1 ? to_f<E>(arow[2 * i + 1]) : 0.0f);
                ar[i] = *reinterpret_cast<const uint32_t*>(&pr);
              }
            }
          }
          // the stored value from an accumulator: alpha acc (SYRK), or
          // fl(cb A + fl(cc acc)) (SQUARE, as ns_stage_kernel rounds it)
          auto value = [&](uint32_t acc_bits, int col) -> float {
            const float y = alpha * __uint_as_float(acc_bits);
            if (kMode != kSquare) return y;
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ar[col >> 1]));
            return fmaf(p.cb, (col & 1) ? f.y : f.x, y);
          };
          uint32_t v0[32], v1[32];
          tmem_ld32(taddr, v0);
          tmem_ld32(taddr + 32, v1);
          tmem_ld_wait();
          if (qi == nq - 1) {
            tc_fence_before();
            mbar_arrive(tempty);            // every TMEM load of the tile has landed
          }
          const int slot = static_cast<int>(gq & 1u);
          uint8_t* rowp = epi + slot * kEpiSlotBytes + row_in_tile * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t wv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int col = c * 8 + 2 * j;
              const float a0 = value(col < 32 ? v0[col] : v1[col - 32], col);
              const float a1 = value(col + 1 < 32 ? v0[col + 1] : v1[col + 1 - 32], col + 1);
              __nv_bfloat162 yv = __floats2bfloat162_rn(a0, a1);
              wv[j] = *reinterpret_cast<uint32_t*>(&yv);
            }
            *reinterpret_cast<uint4*>(rowp + ((c ^ (row_in_tile & 7)) << 4)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
          if (p.diag_full && ti.diag && h == 0 && q >= nq0 / 2) {
            // the diagonal block's upper-right quarter, mirrored into its
            // lower-left one (a warp's lanes are consecutive R: each column
            // is one contiguous run)
            const int R = R0 + row_in_tile;
            if (R < m) {
#pragma unroll
              for (int j = 0; j < 64; ++j) {
                const float a = value(j < 32 ? v0[j] : v1[j - 32], j);
                if (C0 + j < m) A[static_cast<int64_t>(C0 + j) * lda + R] = __float2bfloat16_rn(a);
              }
            }
          }
          fence_proxy_async_smem();
          named_bar_sync(1, 128);
          if (leader) {
            if (R0 < m && C0 < m)
              tma_store_2d(smap, epi + slot * kEpiSlotBytes, C0, R0);
            bulk_commit_group();
            bulk_wait_group_read1();     // the other slot's store has read it
          }
          named_bar_sync(1, 128);        // ... before anyone writes that slot
        }
        continue;
      }
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const bool quarter = ti.diag && h == 1;
        const int R = ti.I * kBN + h * kBM + row_in_tile;
        const int col0 = ti.J * kBN + (quarter ? kBN / 2 : 0);
        const int nch = quarter ? kBN / 64 : kBN / 32;
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q4 * 32) << 16) + static_cast<uint32_t>(h * kBN);
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_ld_wait();
          const int C0 = col0 + c * 32;
          if (R < m && C0 < m && (!p.mirror || C0 + 31 >= R)) {
            float y[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) y[j] = op_round<E>(alpha * __uint_as_float(v[j]));
            E* arow = A + static_cast<int64_t>(R) * lda;
            if (!p.mirror) {
              // the upper triangle and the diagonal 128-blocks, nothing mirrored
              if (C0 + 32 <= m) {
                store32<E>(arow + C0, y);
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (C0 + j < m) arow[C0 + j] = from_f<E>(y[j]);
              }
              if (p.diag_full && ti.diag && h == 0 && c >= nch / 2) {
                // the diagonal block's upper-right quarter, mirrored into its
                // lower-left one (a warp's lanes are consecutive R: each j
                // stores one contiguous run)
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (C0 + j < m) A[static_cast<int64_t>(C0 + j) * lda + R] = from_f<E>(y[j]);
              }
            } else {
              // the whole symmetric A (the quintic SQUARE stage reads all of
              // it): C >= R in place, C > R also at (C, R)
              if (C0 >= R && C0 + 32 <= m) {
                store32<E>(arow + C0, y);
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (C0 + j < m && C0 + j >= R) arow[C0 + j] = from_f<E>(y[j]);
              }
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int C = C0 + j;
                if (C < m && C > R) A[static_cast<int64_t>(C) * lda + R] = from_f<E>(y[j]);
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(tempty);
    }
    if (warp == 2 && lane == 0) bulk_wait_group0();   // the TMA stores have completed
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace dmuon
