// Shared pieces of the persistent grouped GEMMs on sm_100a (5th-generation tensor cores):
// parameters, the tile walker over ragged expert groups, the longest-expert-first order,
// and the fused BF16 epilogues that drain a tensor-memory accumulator (thread = row; two
// warps per 32-lane quadrant, each taking half of the columns).
//
// The kernels that use them (each CTA warp-specialised: warp 0 TMA producer, warp 1 MMA
// issuer, warp 2 tensor-memory allocator, warps 4..11 epilogue; one CTA per SM or one
// 2-CTA cluster per SM pair, walking a static round-robin list of output tiles):
//   grouped_gemm_pair_sm100.cuh         BF16 M-grouped GEMMs on CTA pairs
//   grouped_gemm_kgroup_pair_sm100.cuh  BF16 K-grouped (weight-gradient) GEMMs on pairs
//   grouped_gemm_mxf8_pair_sm100.cuh    MXFP8 M-grouped GEMMs on CTA pairs
//   grouped_gemm_mxf8_sm100.cuh         MXFP8 K-grouped GEMMs on one SM
// Two grouping modes:
//   M-grouped   rows of expert e are [off_e, off_e + n_e) of A and of the output; B is
//               the expert's own [K, N] (or [N, K]) slice. Tiles never straddle two
//               experts in the output: rows past n_e are computed but not stored.
//   K-grouped   (weight gradients) C_e = A_e^T B_e with the contraction over the
//               expert's rows; in the expert's last k-block only the MMA steps holding
//               its rows are issued, and the rows past n_e inside the last partial step
//               are zeroed in shared memory before the MMAs read them.
//
// Pages: "Efficient MoE training for biological foundation models" (sitech.ge section
// "Grouped experts instead of a Python loop"; news.bpdata.com section 1): one grouped
// GEMM over all experts driven by per-expert token counts, and section 3): the fused
// GroupedLinear -> ScaledSwiGLU -> GroupedLinear chain (ScaledSwiGLU is the fc1
// epilogue here) and its backward counterpart.
#pragma once
#include "ptx_sm100.cuh"

namespace moe {

namespace gg {
constexpr int BM = 128;                                  // M of a 1-SM tile (default tile walker rows)
constexpr int BN = 256;                                  // N of an output tile (epilogue column span)
constexpr int BK = 64;                                   // k-block of TileInfo::num_kb (128 bytes of bf16)
constexpr int kMaxE = 1024;                              // experts the kernels' shared tables hold
constexpr uint64_t kTimeoutNs = 4000000000ull;           // 4 s per wait
}  // namespace gg

enum EpiKind : int {
  EPI_STORE = 0,      // out[row, col] = bf16(acc)
  EPI_SWIGLU = 1,     // a = SiLU(g) * u * p  (gate cols of this tile in acc[0:128), up in acc[128:256))
  EPI_DSWIGLU = 2,    // SwiGLU backward from da = acc and the saved h
  EPI_WGRAD = 3,      // out[e, m, n] = bf16(acc), dense per-expert tile
};

struct GemmParams {
  int E;
  int M;                       // M-grouped: total rows R; K-grouped: rows of each expert's output
  int N;                       // output columns (SwiGLU: F, the width of `a`)
  int K;                       // contraction length (M-grouped only)
  const int32_t* split_sizes;  // [E], device
  void* out;                   // bf16 output
  long long ldo;               // elements between output rows
  long long out_batch;         // K-grouped: elements between experts' outputs
  void* out2;                  // SwiGLU: h [R, 2F] (nullable); DSwiGLU: dh [R, 2F]
  long long ldo2;
  const float* probs;          // [R] probability of each permuted row (nullable -> 1)
  const void* aux;             // DSwiGLU: saved h [R, 2F]
  long long ld_aux;
  float* dprob_part;           // DSwiGLU: [2 * ceil(N/256)][R] partial sums (one per N tile half)
  int F;                       // SwiGLU / DSwiGLU: width of the gate half
  int out_f32;                 // EPI_STORE: write fp32 instead of bf16
  uint64_t timeout_ns;         // budget of every wait
  int stall_loads;             // test hook: the producers issue no copies, so the first wait runs out
  // EPI_STORE with the combine fused: row r is added (fp32 vector atomics) into
  // out32[row_token[r]] instead of being stored (out32 [T, ldo] fp32, zeroed beforehand)
  const int32_t* row_token;
  float* out32;
  // STORE (bf16 out): the kernel's output tensor map is valid, so whole 32-row strips
  // inside the expert may be stored by TMA
  int tma_out;
};

// Adds 16 fp32 accumulator values (raw bits) to out32[0..16) with four 16-byte vector
// atomics (sm_90+); the adds into one token's row commute for two terms, so a top-2
// combine is exact and reproducible.
__device__ __forceinline__ void combine_add16(float* out32, const uint32_t* v) {
  float4* d = reinterpret_cast<float4*>(out32);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    atomicAdd(d + i, make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                 __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3])));
}

// Tile decoding shared by the three roles; every role walks the same tile sequence.
struct TileInfo {
  int e;          // expert
  int m_blk, n_blk;
  int row0;       // M-grouped: first row of the tile; K-grouped: first K row of the expert
  int rows;       // M-grouped: valid rows; K-grouped: n_e (length of the contraction)
  int num_kb;     // k-blocks
};

template <bool KGROUP, int TBM = gg::BM>
struct TileWalker {
  static constexpr int kGroupM = 12;   // M-grouped: bound on the m-blocks of a band
  const int32_t* row_off;   // smem [E+1]
  const int32_t* tile_off;  // smem [E+1]
  int E, MT, NT, K;
  const int32_t* order;     // K-grouped: experts by decreasing row count (longest tiles first)
  int cursor = 0;

  __device__ __forceinline__ int total() const { return tile_off[E]; }

  __device__ __forceinline__ TileInfo decode(int t) {
    TileInfo ti;
    if (KGROUP) {
      const int per = MT * NT;
      const int rank = t / per;
      ti.e = order[rank];
      const int local = t - rank * per;
      ti.m_blk = local % MT;
      ti.n_blk = local / MT;
      ti.row0 = row_off[ti.e];
      ti.rows = row_off[ti.e + 1] - row_off[ti.e];
      ti.num_kb = (ti.rows + gg::BK - 1) / gg::BK;
    } else {
      while (tile_off[cursor + 1] <= t) ++cursor;
      ti.e = cursor;
      const int n_e = row_off[ti.e + 1] - row_off[ti.e];
      const int mt = (n_e + TBM - 1) / TBM;
      const int local = t - tile_off[ti.e];
      // grouped order: the expert's m-blocks split into equal bands of at most kGroupM;
      // inside a band every n-block in turn, the band's m-blocks fastest. The tiles in
      // flight at once (one per pair, ~74) then cover about a band's A row blocks and as
      // many B column blocks, which stay in L2 while they are shared, and B streams once
      // per band. An m-fastest walk over a large expert streams all of its A rows once
      // per n-block; fixed bands of 8 left a band of one or two m-blocks at the end of an
      // expert (a Mixtral expert has 8-9) that streamed all of B again for them.
      const int nbands = (mt + kGroupM - 1) / kGroupM;
      const int gsz = (mt + nbands - 1) / nbands;
      const int band = local / (gsz * NT);
      const int gm = min(gsz, mt - band * gsz);
      const int r = local - band * gsz * NT;
      ti.m_blk = band * gsz + r % gm;
      ti.n_blk = r / gm;
      ti.row0 = row_off[ti.e] + ti.m_blk * TBM;
      ti.rows = min(TBM, n_e - ti.m_blk * TBM);
      ti.num_kb = K / gg::BK;
    }
    return ti;
  }
};

// Producer exit of a CTA-pair kernel. Both CTAs' 2-SM copies complete on the leader's
// barriers, so the leader waits (bounded) until the last phase it armed on every ring
// slot has completed — every copy of both CTAs for those stages has landed — and then
// arrives on the second CTA's `drained` barrier. A second CTA whose producer gave up
// waits (bounded) for that arrival before it may leave; on a run without errors the
// leader's waits end as soon as the last stages land.
__device__ __forceinline__ void pair_producer_drain(bool leader, bool ok, uint64_t* drained, uint64_t budget_ns,
                                                    uint64_t* full, int nfull, const ArmedRing& ring,
                                                    uint64_t* full2 = nullptr, int nfull2 = 0,
                                                    const ArmedRing* ring2 = nullptr) {
  if (leader) {
    ring.drain(full, nfull, budget_ns);
    if (ring2) ring2->drain(full2, nfull2, budget_ns);
    mbar_arrive_cluster(map_to_rank(smem_u32(drained), 1));
  } else if (!ok) {
    mbar_wait_drain<true>(drained, 0, budget_ns);
  }
}

// Rank experts by decreasing row count (ties: lower index first) into order[0..E),
// using every thread of the block; row_off must be complete. Static round-robin over
// tiles in this order hands the longest contractions out first.
__device__ __forceinline__ void rank_experts_by_rows(const int32_t* row_off, int E, int32_t* order) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int n = row_off[e + 1] - row_off[e];
    int rank = 0;
    for (int o = 0; o < E; ++o) {
      const int m = row_off[o + 1] - row_off[o];
      rank += (m > n) || (m == n && o < e);
    }
    order[rank] = e;
  }
}

// Drain one BF16 accumulator tile: this thread owns row `tile_row` of the tile (its TMEM
// lane is folded into t_row) and the columns of `half`; applies the fused epilogue EPI.
// A SwiGLU-backward epilogue takes the saved h of its row strip by strip from `h_fetch(g,
// u)` (32 columns of the gate and of the up half, staged in shared memory by the caller in
// the order the strips are drained); other epilogues take none.
struct NoHFetch {
  __device__ bool operator()(uint4 (&)[4], uint4 (&)[4]) const { return false; }
};

// EPI_DSWIGLU: where a warp's dh tiles go by TMA (null stg: lane stores). stg: the warp's
// 2 KB staging tile; tm: dh [R, 2F] bf16 as {2F, R, 1}, boxes {32, 32}, 64-byte swizzle.
struct Bf16Stager {
  uint8_t* stg = nullptr;
  const CUtensorMap* tm = nullptr;
};

// A warp's 32 rows x 32 bf16 (w: this lane's row, starting at global row y) to column x
// by one TMA store through the warp's staging tile (64-byte swizzle: 16-byte chunk j of
// row r at r*64 + 16*(j ^ ((r>>1)&3))); lane 0 first waits until the tile's previous
// store has read it.
__device__ __forceinline__ void store_bf16_tile_tma(uint8_t* stg, const CUtensorMap* tm, int x, int y,
                                                    const uint32_t (&w)[16], int lane) {
  if (lane == 0) bulk_wait_group_read0();
  __syncwarp();
  uint8_t* row = stg + lane * 64;
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4*>(row + 16 * (j ^ sw)) = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_3d(tm, stg, x, y, 0);
    bulk_commit_group();
  }
}

template <int EPI, class HFetch = NoHFetch>
__device__ __forceinline__ void bf16_epilogue_tile(const GemmParams& p, const TileInfo& ti, uint32_t t_row, int half,
                                                   int tile_row, int tile_bm, const HFetch& h_fetch = HFetch{},
                                                   const Bf16Stager& bs = Bf16Stager{}) {
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);

  if (EPI == EPI_STORE || EPI == EPI_WGRAD) {
    const bool zero = (ti.num_kb == 0);
    long long orow;
    bool row_ok;
    if (EPI == EPI_WGRAD) {
      const int m = ti.m_blk * tile_bm + tile_row;
      row_ok = m < p.M;
      orow = (long long)ti.e * p.out_batch + (long long)m * p.ldo;
    } else {
      row_ok = tile_row < ti.rows;
      orow = (long long)(ti.row0 + tile_row) * p.ldo;
    }
    const int n0 = ti.n_blk * gg::BN;
    // 64 columns per round: four tensor-memory loads in flight, one wait
#pragma unroll 1
    for (int c0 = half * (gg::BN / 2); c0 < (half + 1) * (gg::BN / 2); c0 += 64) {
      uint32_t v[4][16];
#pragma unroll
      for (int j = 0; j < 4; ++j) tmem_ld_32x32b_x16(t_row + c0 + 16 * j, v[j]);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = c0 + 16 * j;
        if (!row_ok || n0 + c >= p.N) continue;
        if (EPI == EPI_STORE && p.row_token) {
          combine_add16(p.out32 + (long long)p.row_token[ti.row0 + tile_row] * p.ldo + n0 + c, v[j]);
        } else if (EPI == EPI_STORE && p.out_f32) {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<float*>(p.out) + orow + n0 + c);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(v[j][4 * i], v[j][4 * i + 1], v[j][4 * i + 2], v[j][4 * i + 3]);
        } else {
          uint4 o[2];
          uint32_t* ow = reinterpret_cast<uint32_t*>(o);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            ow[i] = zero ? 0u : pack_bf16x2(__uint_as_float(v[j][2 * i]), __uint_as_float(v[j][2 * i + 1]));
          uint4* dst = reinterpret_cast<uint4*>(out + orow + n0 + c);
          dst[0] = o[0];
          dst[1] = o[1];
        }
      }
    }
  } else if (EPI == EPI_SWIGLU) {
    const bool row_ok = tile_row < ti.rows;
    const long long row = ti.row0 + tile_row;
    const float pr = (row_ok && p.probs) ? p.probs[row] : 1.0f;
    const int n0 = ti.n_blk * 128;
    __nv_bfloat16* hout = reinterpret_cast<__nv_bfloat16*>(p.out2);
#pragma unroll 1
    for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
      // 32 columns per round: four tensor-memory loads in flight, one wait
      uint32_t gg2[2][16], uu2[2][16];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        tmem_ld_32x32b_x16(t_row + c0 + 16 * j, gg2[j]);
        tmem_ld_32x32b_x16(t_row + 128 + c0 + 16 * j, uu2[j]);
      }
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int c = c0 + 16 * j;
        const uint32_t* g = gg2[j];
        const uint32_t* u = uu2[j];
        if (row_ok) {
          uint4 o[2];
          uint32_t* ow = reinterpret_cast<uint32_t*>(o);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
            const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
            ow[i] = pack_bf16x2(silu_f(g0) * u0 * pr, silu_f(g1) * u1 * pr);
          }
          uint4* dst = reinterpret_cast<uint4*>(out + row * p.ldo + n0 + c);
          dst[0] = o[0];
          dst[1] = o[1];
          if (hout) {
            uint4 hg[2], hu[2];
            uint32_t* hgw = reinterpret_cast<uint32_t*>(hg);
            uint32_t* huw = reinterpret_cast<uint32_t*>(hu);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              hgw[i] = pack_bf16x2(__uint_as_float(g[2 * i]), __uint_as_float(g[2 * i + 1]));
              huw[i] = pack_bf16x2(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1]));
            }
            uint4* hd = reinterpret_cast<uint4*>(hout + row * p.ldo2 + n0 + c);
            hd[0] = hg[0];
            hd[1] = hg[1];
            uint4* hd2 = reinterpret_cast<uint4*>(hout + row * p.ldo2 + p.F + n0 + c);
            hd2[0] = hu[0];
            hd2[1] = hu[1];
          }
        }
      }
    }
  } else if (EPI == EPI_DSWIGLU) {
    // acc = da for columns [n0, n0+256) of F; h = [g | u] saved by the forward
    const bool row_ok = tile_row < ti.rows;
    const long long row = ti.row0 + tile_row;
    const float pr = (row_ok && p.probs) ? p.probs[row] : 1.0f;
    __nv_bfloat16* dh = reinterpret_cast<__nv_bfloat16*>(p.out2);
    const int n0 = ti.n_blk * gg::BN;
    const int lane = threadIdx.x & 31;
    // the warp's 32 rows all belong to the expert: its dg / du tiles go by TMA
    const int w_row = tile_row - lane;
    const bool tma = bs.stg != nullptr && w_row + 32 <= ti.rows;   // warp-uniform
    float dp = 0.f;
#pragma unroll 1
    for (int c0 = half * (gg::BN / 2); c0 < (half + 1) * (gg::BN / 2); c0 += 32) {
      // 32 columns per round; the saved h of the round comes from shared memory (every
      // round takes its strip, so that the staging ring advances in step), before the
      // tensor-memory loads: nothing may run between a tcgen05.ld and its wait
      uint4 gva[4], uva[4];
      const bool cols_ok0 = row_ok && n0 + c0 < p.N;
      const bool cols_ok1 = row_ok && n0 + c0 + 16 < p.N;
      h_fetch(gva, uva);
      uint32_t vv[2][16];
      tmem_ld_32x32b_x16(t_row + c0, vv[0]);
      tmem_ld_32x32b_x16(t_row + c0 + 16, vv[1]);
      tmem_wait_ld();
      uint32_t ogw[16], ouw[16];   // this row's 32 dg and 32 du, bf16 pairs
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const uint32_t* v = vv[jj];
        if (jj == 0 ? cols_ok0 : cols_ok1) {
          const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(gva + 2 * jj);
          const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(uva + 2 * jj);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float2 gg2 = __bfloat1622float2(g2[i]);
            const float2 uu2 = __bfloat1622float2(u2[i]);
            float dg[2], du[2];
            const float gs[2] = {gg2.x, gg2.y}, us[2] = {uu2.x, uu2.y};
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const float da = __uint_as_float(v[2 * i + j]);
              const float sg = sigmoid_f(gs[j]);
              const float sl = gs[j] * sg;
              dg[j] = da * pr * us[j] * (sg * (1.0f + gs[j] * (1.0f - sg)));
              du[j] = da * pr * sl;
              dp = fmaf(da, sl * us[j], dp);
            }
            ogw[8 * jj + i] = pack_bf16x2(dg[0], dg[1]);
            ouw[8 * jj + i] = pack_bf16x2(du[0], du[1]);
          }
        }
      }
      if (tma && n0 + c0 + 32 <= p.N) {   // warp-uniform
        store_bf16_tile_tma(bs.stg, bs.tm, n0 + c0, (int)(ti.row0 + w_row), ogw, lane);
        store_bf16_tile_tma(bs.stg, bs.tm, p.F + n0 + c0, (int)(ti.row0 + w_row), ouw, lane);
      } else {
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          if (!(jj == 0 ? cols_ok0 : cols_ok1)) continue;
          const int c = c0 + 16 * jj;
          uint4* dg_dst = reinterpret_cast<uint4*>(dh + row * p.ldo2 + n0 + c);
          dg_dst[0] = make_uint4(ogw[8 * jj], ogw[8 * jj + 1], ogw[8 * jj + 2], ogw[8 * jj + 3]);
          dg_dst[1] = make_uint4(ogw[8 * jj + 4], ogw[8 * jj + 5], ogw[8 * jj + 6], ogw[8 * jj + 7]);
          uint4* du_dst = reinterpret_cast<uint4*>(dh + row * p.ldo2 + p.F + n0 + c);
          du_dst[0] = make_uint4(ouw[8 * jj], ouw[8 * jj + 1], ouw[8 * jj + 2], ouw[8 * jj + 3]);
          du_dst[1] = make_uint4(ouw[8 * jj + 4], ouw[8 * jj + 5], ouw[8 * jj + 6], ouw[8 * jj + 7]);
        }
      }
    }
    if (row_ok) p.dprob_part[(long long)(2 * ti.n_blk + half) * p.M + row] = dp;
  }
}

// dprobs_perm[r] = sum over n-tiles (in order) of the DSwiGLU partial sums.
__global__ void reduce_dprob_kernel(const float* __restrict__ part, int nparts, int R, float* __restrict__ out) {
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < R; r += gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int i = 0; i < nparts; ++i) s += part[(long long)i * R + r];
    out[r] = s;
  }
}

}  // namespace moe
