// GEMM stage of the batched Muon update on CTA pairs (sm_100a): X' = c (a X +
// b A X) (quintic: c (a X + P X)) over 256 x 256 output tiles, each computed
// by a two-CTA cluster with pair UMMAs (tcgen05 cta_group::2), for every
// matrix of a bf16 group.
//
// Source: DMuon blog post "DMuon：让矩阵正交化优化器达到接近 AdamW 的分布式训练开销",
// section "Muon 核心：Newton-Schulz 迭代" (the cubic step X <- a X + b A X).
// Included by kernels.cuh after ns_stage.cuh, whose epilogue it shares.
#pragma once

namespace dmuon {
// ======================================================================
// A pair tile covers rows 256 I .. 256 I + 255 and columns 256 J .. of X'.
// CTA r of the cluster (r = 0, 1) owns rows 256 I + 128 r .. + 127: per
// k-block it loads those 128 rows of A (16 KB) and columns 256 J + 128 r ..
// + 127 of X (16 KB, MN-major), and its TMEM receives its 128 rows x 256
// columns of A X.  The even CTA issues every UMMA (M = 256, N = 256); it
// reads the odd CTA's operands at the same shared-memory offsets.  Each SM
// thus brings and reads 32 KB of operands per 128 x 256 x 64 of work,
// against 48 KB for a 128 x 256 tile on one SM, and the 192 KB ring holds six
// stages instead of four.
//
// Both CTAs' TMA loads (pair form, no multicast) complete on the even CTA's
// `full` barrier, which the even CTA arms for both CTAs' bytes.  UMMA
// completion arrives on `empty` (stage free) and `tfull` (accumulator ready)
// in both CTAs at once; both CTAs' epilogue warps release an accumulator
// buffer on the even CTA's `tempty`.  Producer, UMMA and epilogue waits poll
// (their signals come from the other SM).
//
// A (or P) is read as the SYRK (or the quintic SQUARE stage) stored it:
// upper triangle plus full diagonal 256-blocks.  The k-blocks left of the
// pair's diagonal block come transposed (MN-major) from the upper triangle,
// as in ns_stage_kernel.
// ======================================================================
constexpr int kG2Stages = 6;
constexpr int kG2ABytes = kBM * 128;            // 128 rows (or 128 M columns) x 128 bytes of K
constexpr int kG2BBytes = (kBN / 2) * 128;      // 128 columns x 64 K rows, MN-major
constexpr int kG2StageBytes = kG2ABytes + kG2BBytes;
constexpr int kG2SmemBytes = kG2Stages * kG2StageBytes + kEpiSlots * kEpiSlotBytes + 1024 /*align*/ + 256;
static_assert(kG2SmemBytes <= 232448, "exceeds the 227 KB of shared memory per block");
constexpr uint32_t kG2TemptyArrivals = 2 * 4;  // one per epilogue warp of both CTAs

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kNsThreads, 1)
    gemm_pair_kernel(const __grid_constant__ NsParams p) {
  using E = __nv_bfloat16;
  constexpr int BK = 64;          // K elements per stage (one 128-byte row)
  constexpr int MMA_K = 16;       // K per UMMA instruction
  constexpr int KSTEPS = BK / MMA_K;
  constexpr uint32_t IDESC = make_idesc(1u, 0u, 1u, 2 * kBM, kBN);      // A K-major, X MN-major
  constexpr uint32_t IDESC_AT = make_idesc(1u, 1u, 1u, 2 * kBM, kBN);   // A k-block transposed

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  // stage s: A part at s * 32 KB, this CTA's half of the X part 16 KB after it
  uint8_t* epi = smem + kG2Stages * kG2StageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi + kEpiSlots * kEpiSlotBytes);   // even CTA's used
  uint64_t* empty = full + kG2Stages;
  uint64_t* tfull = empty + kG2Stages;
  uint64_t* tempty = tfull + 2;            // even CTA's is the one used
  uint64_t* xfull = tempty + 2;            // [kEpiSlots]
  uint64_t* drain = xfull + kEpiSlots;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(cluster_id_x());
  const int npairs = static_cast<int>(cluster_count_x());

  if (threadIdx.x == 0) {
    for (int s = 0; s < kG2Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kG2TemptyArrivals);
    }
    for (int e = 0; e < kEpiSlots; ++e) mbar_init(&xfull[e], 1);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, kTmemCols);
    tmem_relinquish_pair();
  }
  // Both CTAs' barriers are initialised before either CTA arrives on the
  // other's.
  tc_fence_before();
  cluster_sync_all();
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
    // ------------------------------------------------ TMA producer (both CTAs)
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_phase[kG2Stages];
    bool issued[kG2Stages];
#pragma unroll
    for (int s = 0; s < kG2Stages; ++s) { issued[s] = false; issued_phase[s] = 0; }
    int fenced = -1;
    for (int t = pair; t < p.ntiles && ok; t += npairs) {
      const TileInfo ti = decode_tile<kGemm, BK, true>(p, t, static_cast<int>(rank));
      const MatMaps& mp = p.maps[ti.mi];
      const CUtensorMap* mapA = p.quintic ? &mp.p : &mp.a;
      const CUtensorMap* mapAt = p.quintic ? &mp.pmn : &mp.amn;
      const CUtensorMap* mapB = &mp.xmn2[p.cur];
      // k-blocks left of the pair's diagonal 256-block: A transposed
      const int kb_t = p.a_upper ? (ti.tm >> 1) * (2 * kBM / BK) : 0;
      if (lane == 0 && ti.mi != fenced) {
        tensormap_acquire_gpu(mapA);
        tensormap_acquire_gpu(mapB);
        if (p.a_upper) tensormap_acquire_gpu(mapAt);
        fenced = ti.mi;
      }
      for (int kb = 0; kb < ti.nkb; ++kb) {
        bool w = mbar_wait_spin(&empty[stage], phase ^ 1u, p.err, p.wait_limit_ns);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        if (lane == 0) {
          // Both CTAs' loads complete on the even CTA's barrier, which the
          // even CTA arms for both.
          const uint32_t bar0 = mapa_shared(&full[stage], 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * kG2StageBytes);
          uint8_t* a_dst = smem + stage * kG2StageBytes;
          if (kb < kb_t) {
            // this CTA's 128 M columns in two 128-byte chunks, BK rows of K each
            tma_load_2d_pair(a_dst, mapAt, bar0, ti.tm * kBM, kb * BK);
            tma_load_2d_pair(a_dst + BK * 128, mapAt, bar0, ti.tm * kBM + 64, kb * BK);
          } else {
            tma_load_2d_pair(a_dst, mapA, bar0, kb * BK, ti.tm * kBM);
          }
          // column blocks 4 J + 2 r and 4 J + 2 r + 1 of X (past the last
          // column they arrive as zeros)
          tma_load_3d_pair(a_dst + kG2ABytes, mapB, bar0, 0, kb * BK,
                           ti.tn * (kBN / 64) + 2 * static_cast<int>(rank));
        }
        __syncwarp();
        issued[stage] = true;
        issued_phase[stage] = phase;
        if (++stage == kG2Stages) { stage = 0; phase ^= 1u; }
      }
    }
    if (ok) {
      // Every stage's last release (a UMMA commit from the even CTA) has
      // arrived before this CTA may leave.
      for (int i = 0; i < kG2Stages && ok; ++i) {
        ok = __all_sync(0xffffffffu, mbar_wait_spin(&empty[stage], phase ^ 1u, p.err, p.wait_limit_ns));
        if (++stage == kG2Stages) { stage = 0; phase ^= 1u; }
      }
    } else if (lane == 0 && rank == 0) {
      // Let every load already issued land before the CTA's memory goes away.
      for (int s = 0; s < kG2Stages; ++s)
        if (issued[s]) mbar_wait_spin(&full[s], issued_phase[s], nullptr, p.wait_limit_ns, 1024);
    } else if (lane == 0) {
      // The odd CTA's loads complete on the even CTA's barriers: give them
      // 100 microseconds to land before this CTA's memory goes away.
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 100000u) __nanosleep(1000);
    }
  } else if (warp == 1 && rank == 0) {
    // ------------------------------------------------ even CTA: pair UMMA issuer
    // (the odd CTA's warp 1 only allocates and frees TMEM)
    int stage = 0;
    uint32_t phase = 0;
    int lt = 0;
    for (int t = pair; t < p.ntiles && ok; t += npairs, ++lt) {
      const TileInfo ti = decode_tile<kGemm, BK, true>(p, t, 0);
      const int b = lt & 1;
      const uint32_t tph = (static_cast<uint32_t>(lt) >> 1) & 1u;
      bool w = mbar_wait_spin(&tempty[b], tph ^ 1u, p.err, p.wait_limit_ns);
      if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * kBN);
      const int kb_t = p.a_upper ? (ti.tm >> 1) * (2 * kBM / BK) : 0;
      for (int kb = 0; kb < ti.nkb; ++kb) {
        w = mbar_wait_spin(&full[stage], phase, p.err, p.wait_limit_ns);
        if (!__all_sync(0xffffffffu, w)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_base = smem_u32(smem + stage * kG2StageBytes);
          const uint32_t b_base = a_base + kG2ABytes;
          const bool at = kb < kb_t;
#pragma unroll
          for (int k = 0; k < KSTEPS; ++k) {
            const uint64_t ad = at ? sw128_desc(a_base + k * MMA_K * 128, BK * 128, 1024, kSwizzle128B)
                                   : sw128_desc(a_base + k * 32, 16, 1024);
            const uint64_t bd = sw128_desc(b_base + k * MMA_K * 128, BK * 128, 1024, kSwizzle128B);
            umma_f16_pair(d_tmem, ad, bd, at ? IDESC_AT : IDESC, (kb > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit_pair_mc(&empty[stage], 0x3);
        }
        __syncwarp();
        if (++stage == kG2Stages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (lane == 0) umma_commit_pair_mc(&tfull[b], 0x3);
      __syncwarp();
    }
    if (ok) {
      // Both CTAs' epilogues have released both accumulator buffers (their
      // arrivals on this CTA's barriers have landed).
      for (int i = 0; i < 2 && ok; ++i, ++lt) {
        const uint32_t tph = (static_cast<uint32_t>(lt) >> 1) & 1u;
        ok = __all_sync(0xffffffffu, mbar_wait_spin(&tempty[lt & 1], tph ^ 1u, p.err, p.wait_limit_ns));
      }
    } else if (lane == 0) {
      // Wait for every UMMA this thread issued before TMEM is released.
      umma_commit_pair(drain);
      mbar_wait_spin(drain, 0, nullptr, p.wait_limit_ns, 1024);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------ epilogue (4 warps, both CTAs)
    ok = run_epilogue<kGemm, E, true>(p, tmem_base, epi, tfull, xfull, warp, lane, pair, npairs,
                                [&](int b) {
                                  tc_fence_before();
                                  __syncwarp();
                                  if (lane == 0) mbar_arrive_cluster(mapa_shared(&tempty[b], 0));
                                },
                                static_cast<int>(rank));
  }

  // Neither CTA leaves (or frees TMEM) while the other may still arrive on
  // its barriers or, for the even CTA, write its TMEM.
  __syncthreads();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace dmuon
