// MXFP8 weight-gradient GEMMs on a pair of SMs (tcgen05.mma.cta_group::2.kind::mxf8f6f4
// .block_scale), K-grouped: dW[e] = A_e^T B_e with the contraction over expert e's rows.
// A_e [n_e, M] and B_e [n_e, N] are E4M3 (or E5M2) codes, MN-major (their rows are K),
// quantised along the rows with one E8M0 scale per 32 rows of one column, the blocks
// restarting at every expert.
//
// Pages: "Efficient MoE training for biological foundation models" (news.bpdata.com
// section 2: MXFP8 operands whose scales the tensor cores consume directly; section 3: the
// backward of the fused GroupedLinear chain, whose weight gradients are grouped GEMMs over
// each expert's tokens).
//
// Why pairs: a 1-SM 128 x 256 tile needs 48 KB of operands per 128 K rows for 8.4 MFLOP;
// a 256 x 256 pair tile needs 32 KB per CTA for the same work per SM, two thirds of the
// L2 -> SM traffic, which the M-grouped pair GEMMs showed the tensor pipe needs.
//
// Layout (per CTA): a k-stage is 256 K rows (two 128-row k-groups): ONE copy per operand
// brings this CTA's 128 columns of A and its half (128 columns) of B, box {128 bytes,
// 256 rows}, 128-byte swizzle, 32 KB each, three stages. Scale atoms (512 bytes: 128
// columns x four 32-row blocks of one k-group, column c at word (c % 32) * 4 + c / 32)
// travel on their own two-slot ring, four k-groups per copy: this CTA's A column group and
// both column groups of the B tile (the block-scaled pair MMA reads every N column's
// scales from each CTA's own tensor memory). Atom (cg, kg) of expert e sits at
// kg_off[e] * (C / 128) + cg * KG_e + kg; a copy that runs past the expert's last k-group
// reads atoms the MMAs never use, and past the end of the buffer zeros.
//
// The last stage of an expert is ragged: its rows past n_e belong to the next expert and
// must not contribute. The leader issues only the K=32 steps that hold the expert's rows;
// inside the last partial step both CTAs zero their own rows past n_e. As in the BF16
// weight-gradient pair kernel, for that one stage both CTAs load with the 1-SM form onto
// their own barriers; the second CTA's warp 1 zeroes and signals the leader's `rready`.
//
// Tensor memory per CTA: overlapping accumulators acc0 = [0, 256) and acc1 = [192, 448),
// four scale sets at 448..495 that warp 2 of the leader fills ahead of the MMA thread
// (the M-grouped MXFP8 layout, ScaleCopier). Waits are bounded.
#pragma once
#include "grouped_gemm_mxf8_pair_sm100.cuh"

namespace moe {

namespace mkp {
constexpr int BM = 256;                       // M of a pair tile (128 per CTA)
constexpr int BMC = 128;
constexpr int BN = 256;                       // N of a pair tile (128 per CTA)
constexpr int kGroupsPerStage = 2;            // 128-row k-groups per stage
constexpr int BK = 128 * kGroupsPerStage;     // K rows per stage
constexpr int kStages = 3;
constexpr int kThreads = 384;
constexpr int kABytes = 128 * BK;             // this CTA's 128 columns of A, 32 KB
constexpr int kBBytes = 128 * BK;             // this CTA's 128 columns of B, 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kSfKg = 4;                      // k-groups per scale copy
constexpr int kSfGroupBytes = kSfKg * 512;
constexpr int kSfSlotBytes = 3 * kSfGroupBytes;   // A group, B lower group, B upper group
constexpr int kSfSlots = 2;
constexpr int kStPerSf = kSfKg / kGroupsPerStage;
constexpr int kMaxE = 1024;
constexpr int kTmemCols = 512;
constexpr int kSmemBytes =
    1024 + kStages * kStageBytes + kSfSlots * kSfSlotBytes + 1024 + 4 * (kMaxE + 1) * 4;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
// ScaleCopier's look-back of mx::kSfSets k-groups must stay within the operand ring
static_assert(mx::kSfSets <= kStages * kGroupsPerStage, "operand ring too short for the scale-set look-back");
}  // namespace mkp

// Zero rows [valid, end) of this CTA's A and B blocks of one stage (128-byte rows), one
// warp; then make the stores visible to the tensor cores' reads.
__device__ __forceinline__ void mkp_zero_rows(uint8_t* a_st, uint8_t* b_st, int valid, int end, int lane) {
  const int zr = end - valid;
  if (zr > 0) {
    for (int i = lane; i < 2 * zr * 8; i += 32) {
      const int v = i & 7, rb = i >> 3;
      const int blk = rb / zr, r = rb - blk * zr;
      uint8_t* base = blk == 0 ? a_st : b_st;
      *reinterpret_cast<uint4*>(base + (valid + r) * 128 + v * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  __syncwarp();
}

// tmA: A codes [R, M] as {M, R, 1}, box {128, 256}; tmB: B codes [R, N] likewise.
// tmSa / tmSb: the grouped scale atoms of A / B as uint32 {128 words, atoms, 1}, box {128,
// 4}. Output dW[e] [M, N] bf16 at p.out + e * p.out_batch.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(mkp::kThreads, 1)
    grouped_wgrad_mxf8_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                   const __grid_constant__ CUtensorMap tmSa, const __grid_constant__ CUtensorMap tmSb,
                                   const MxGemmParams mp) {
  using namespace mkp;
  const GemmParams& p = mp.g;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + kStages * kABytes;
  uint8_t* sSf = sB + kStages * kBBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSf + kSfSlots * kSfSlotBytes);
  uint64_t* full = bars;                       // leader: 2-SM copies, and its own copies of a ragged stage
  uint64_t* empty = bars + kStages;            // both CTAs
  uint64_t* pfull = bars + 2 * kStages;        // second CTA: its own copies of a ragged stage
  uint64_t* rready = bars + 3 * kStages;       // leader: the second CTA has zeroed its ragged stage
  uint64_t* tfull = bars + 4 * kStages;        // both CTAs
  uint64_t* tempty = tfull + 2;                // leader
  uint64_t* tovl = tempty + 2;                 // leader
  uint64_t* sfull = tovl + 1;                  // scale ring: leader
  uint64_t* sempty = sfull + kSfSlots;         // scale ring: both CTAs
  uint64_t* drained = sempty + kSfSlots;       // second CTA
  uint64_t* setfull = drained + 1;             // tensor-memory scale sets: leader
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(setfull + mx::kSfSets);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* row_off = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(bars) + 1024);
  int32_t* tile_off = row_off + (kMaxE + 1);
  int32_t* kg_off = tile_off + (kMaxE + 1);   // 128-row k-groups of earlier experts
  int32_t* order = kg_off + (kMaxE + 1);      // experts by decreasing row count

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int E = p.E;
  const int MT = (p.M + BM - 1) / BM, NT = (p.N + BN - 1) / BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&pfull[s], 1);
      mbar_init(&rready[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 16);   // 8 epilogue warps in each CTA of the pair
    }
    mbar_init(tovl, 16);
    for (int s2 = 0; s2 < kSfSlots; ++s2) {
      mbar_init(&sfull[s2], 1);
      mbar_init(&sempty[s2], 1);
    }
    mbar_init(drained, 1);
    for (int b = 0; b < mx::kSfSets; ++b) {
      mbar_init(&setfull[b], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmSa);
    tma_prefetch_desc(&tmSb);
  }
  if (warp == 3) {
    int carry_r = 0, carry_t = 0, carry_k = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int n = (e < E) ? p.split_sizes[e] : 0;
      const int tiles = (e < E) ? MT * NT : 0;
      const int kgs = (n + 127) / 128;
      int ir = n, it = tiles, ik = kgs;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yr = __shfl_up_sync(0xffffffffu, ir, o);
        const int yt = __shfl_up_sync(0xffffffffu, it, o);
        const int yk = __shfl_up_sync(0xffffffffu, ik, o);
        if (lane >= o) {
          ir += yr;
          it += yt;
          ik += yk;
        }
      }
      if (e < E) {
        row_off[e] = carry_r + ir - n;
        tile_off[e] = carry_t + it - tiles;
        kg_off[e] = carry_k + ik - kgs;
      }
      carry_r += __shfl_sync(0xffffffffu, ir, 31);
      carry_t += __shfl_sync(0xffffffffu, it, 31);
      carry_k += __shfl_sync(0xffffffffu, ik, 31);
    }
    if (lane == 0) {
      row_off[E] = carry_r;
      tile_off[E] = carry_t;
      kg_off[E] = carry_k;
    }
  }
  if (warp == 2) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  rank_experts_by_rows(row_off, E, order);
  __syncthreads();
  cluster_sync();   // both CTAs' barriers are initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  TileWalker<true, BM> walk{row_off, tile_off, E, MT, NT, p.K, order};
  const int total = walk.total();
  auto stages_of = [](const TileInfo& ti) { return (ti.rows + BK - 1) / BK; };
  auto ragged = [](const TileInfo& ti, int st, int nst) { return st == nst - 1 && (ti.rows % BK) != 0; };

  if (warp == 0) {
    // ---------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0, sslot = 0;
      uint32_t phase = 0, sphase = 0;
      ArmedRing ring, pring, sring;   // leader: full, sfull; second CTA: its ragged-stage pfull
      bool ok = true;
      const int cga_n = p.M / 128, cgb_n = p.N / 128;   // column groups of A and B
      for (int t = pair; t < total && ok && !p.stall_loads; t += npairs) {
        const TileInfo ti = walk.decode(t);
        const int nst = stages_of(ti);
        const int kge = (ti.rows + 127) / 128;
        // this CTA's 128 columns of A and of B; the B tile's two column groups (a group
        // past N reads codes of zeros and atoms the epilogue's stores never reach)
        const int ma = ti.m_blk * BM + BMC * (int)rank;
        const int nb = ti.n_blk * BN + 128 * (int)rank;
        const int ga = kg_off[ti.e] * cga_n + (ma / 128) * kge;
        const int gb0 = kg_off[ti.e] * cgb_n + (ti.n_blk * 2) * kge;
        const int gb1 = gb0 + kge;
        for (int st = 0; st < nst; ++st) {
          if (st % kStPerSf == 0) {
            if (!mbar_wait_bounded(&sempty[sslot], sphase ^ 1, abort_flag, p.timeout_ns)) {
              ok = false;
              break;
            }
            if (leader) {
              mbar_arrive_expect_tx(&sfull[sslot], 2 * kSfSlotBytes);
              sring.arm(sslot, sphase);
            }
            uint8_t* sd = sSf + sslot * kSfSlotBytes;
            const int kg = kGroupsPerStage * st;
            tma_load_3d_pair(sd, &tmSa, &sfull[sslot], 0, ga + kg, 0);
            tma_load_3d_pair(sd + kSfGroupBytes, &tmSb, &sfull[sslot], 0, gb0 + kg, 0);
            tma_load_3d_pair(sd + 2 * kSfGroupBytes, &tmSb, &sfull[sslot], 0, gb1 + kg, 0);
            if (++sslot == kSfSlots) {
              sslot = 0;
              sphase ^= 1;
            }
          }
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          const int k0 = ti.row0 + st * BK;
          if (!ragged(ti, st, nst)) {
            if (leader) {
              mbar_arrive_expect_tx(&full[stage], 2 * kStageBytes);
              ring.arm(stage, phase);
            }
            tma_load_3d_pair(sA + stage * kABytes, &tmA, &full[stage], ma, k0, 0);
            tma_load_3d_pair(sB + stage * kBBytes, &tmB, &full[stage], nb, k0, 0);
          } else {
            // ragged last stage: each CTA's copies land on its own barrier, so that it can
            // zero its rows past the expert before the MMAs read them
            uint64_t* bar = leader ? &full[stage] : &pfull[stage];
            mbar_arrive_expect_tx(bar, kStageBytes);
            (leader ? ring : pring).arm(stage, phase);
            tma_load_3d(sA + stage * kABytes, &tmA, bar, ma, k0, 0);
            tma_load_3d(sB + stage * kBBytes, &tmB, bar, nb, k0, 0);
          }
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!leader && !ok) pring.drain(pfull, kStages, p.timeout_ns);
      pair_producer_drain(leader, ok, drained, p.timeout_ns, full, kStages, ring, sfull, kSfSlots, &sring);
    }
  } else if (warp == 1 && !leader) {
    // -------------------- second CTA: zero its rows of each ragged stage, tell the leader
    const uint32_t rready_leader0 = map_to_rank(smem_u32(&rready[0]), 0);
    int stage = 0;
    uint32_t pmask = 0;   // phase parity of pfull per ring slot
    bool ok = true;
    for (int t = pair; t < total && ok; t += npairs) {
      const TileInfo ti = walk.decode(t);
      const int nst = stages_of(ti);
      for (int st = 0; st < nst; ++st) {
        if (ragged(ti, st, nst)) {
          if (!mbar_wait_bounded(&pfull[stage], (pmask >> stage) & 1u, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          pmask ^= 1u << stage;
          const int valid = ti.rows - st * BK;
          mkp_zero_rows(sA + stage * kABytes, sB + stage * kBBytes, valid, (valid + 31) / 32 * 32, lane);
          if (lane == 0) mbar_arrive_cluster(rready_leader0 + stage * 8);
        }
        if (++stage == kStages) stage = 0;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (pair leader)
    int stage = 0;
    uint32_t phase = 0, rmask = 0;
    int lt = 0;
    bool ok = true;
    ScaleSets sets{setfull, tmem_base};
    for (int t = pair; t < total && ok; t += npairs, ++lt) {
      const TileInfo ti = walk.decode(t);
      const int nst = stages_of(ti);
      const int acc = lt & 1;
      if (!mbar_wait_bounded<true>(&tempty[acc], ((lt >> 1) & 1) ^ 1, abort_flag, p.timeout_ns)) break;
      if (lt > 0 && !mbar_wait_bounded<true>(tovl, (lt - 1) & 1, abort_flag, p.timeout_ns)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (acc ? mx::kAcc1Col : 0u);
      for (int st = 0; st < nst && ok; ++st) {
        if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        int ksteps = BK / 32;   // K=32 MMAs of this stage
        if (ragged(ti, st, nst)) {
          // MMAs only over the expert's rows; zero this CTA's rows inside the last partial
          // step, then wait until the second CTA has done the same with its rows
          const int valid = ti.rows - st * BK;
          ksteps = (valid + 31) / 32;
          mkp_zero_rows(sA + stage * kABytes, sB + stage * kBBytes, valid, ksteps * 32, lane);
          if (!mbar_wait_bounded<true>(&rready[stage], (rmask >> stage) & 1u, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          rmask ^= 1u << stage;
          tc_fence_after();
        }
        const uint32_t a_addr = smem_u32(sA + stage * kABytes);
        const uint32_t b_addr = smem_u32(sB + stage * kBBytes);
        for (int c = 0; c < kGroupsPerStage; ++c) {
          if (4 * c >= ksteps) break;
          // this k-group's scale atoms, copied into tensor memory by the scale warp
          if (!sets.wait(abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t sfa = sets.sfa(), sfb = sets.sfb();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              if (4 * c + kk < ksteps) {
                // MN-major: 32 k rows = 4096 bytes further (four 8-row swizzle atoms)
                const uint32_t off = (uint32_t)(4 * c + kk) * 4096;
                const uint64_t adesc = make_sdesc(a_addr + off, kABytes, 1024, 2);
                const uint64_t bdesc = make_sdesc(b_addr + off, kBBytes, 1024, 2);
                const uint32_t idesc = make_idesc_mxf8(BM, BN, true, true, kk, kk) | mp.ab_fmt;
                mma_mxf8_pair(d_tmem, adesc, bdesc, idesc, sfa | ((uint32_t)kk << 30), sfb | ((uint32_t)kk << 30),
                              (st > 0 || c > 0 || kk > 0) ? 1u : 0u);
              }
            }
          }
          sets.next();
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) mma_commit_pair(&empty[stage]);
        __syncwarp();
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      // (an expert without rows: no MMAs, the commit arrives once the earlier ones are
      // done and the epilogue writes zeros)
      if (lane == 0) mma_commit_pair(&tfull[acc]);
      __syncwarp();
    }
  } else if (warp == 2) {
    // ------------------------------------ scale copies (pair leader): every k-group's
    // atoms into the next tensor-memory scale set, ahead of the MMA thread
    if (leader && lane == 0) {
      ScaleCopier<kSfKg> cp{sfull, sempty, setfull, empty, kStages, sSf, kSfSlots, tmem_base, abort_flag, p.timeout_ns};
      bool ok = true;
      int g0 = 0;   // global stage of the tile's first k-group
      for (int t = pair; t < total && ok; t += npairs) {
        const TileInfo ti = walk.decode(t);
        const int nkg = (ti.rows + 127) / 128;   // k-groups holding the expert's rows
        for (int kg = 0; kg < nkg && ok; ++kg) ok = cp.copy(kg, kg == nkg - 1, g0 + kg / kGroupsPerStage);
        g0 += stages_of(ti);
      }
      cp.drain();
    }
  } else if (warp >= 4) {
    // -------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r_local = q * 32 + lane;
    const uint32_t tempty_leader0 = map_to_rank(smem_u32(&tempty[0]), 0);
    const uint32_t tovl_leader = map_to_rank(smem_u32(tovl), 0);
    int lt = 0;
    for (int t = pair; t < total; t += npairs, ++lt) {
      const TileInfo ti = walk.decode(t);
      const int acc = lt & 1;
      if (!mbar_wait_bounded(&tfull[acc], (lt >> 1) & 1, abort_flag, p.timeout_ns)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (acc ? mx::kAcc1Col : 0u) + ((uint32_t)(q * 32) << 16);
      mxf8_epilogue_tile<MXEPI_WGRAD>(mp, ti, t_row, acc, half, BMC * (int)rank + r_local, BM, [&] {
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tovl_leader);
      });
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + acc * 8);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // neither CTA leaves while the other can still signal it
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace moe
