// Persistent grouped GEMM for sm_100a on the 5th-generation tensor cores.
//
// One CTA per SM walks a static round-robin list of output tiles spread over ragged
// expert groups. Inside a CTA the work is warp-specialised:
//   warp 0      TMA producer: fills a ring of kStages shared-memory stages;
//   warp 1      MMA issuer: one thread issues tcgen05.mma (M=128, N=256, K=16 for
//               bf16) into one of two tensor-memory accumulators (2 x 256 fp32 columns);
//   warp 2      tensor-memory allocator;
//   warps 4..11 epilogue: tcgen05.ld the accumulator (thread = row; two warps per
//               32-lane quadrant, each taking half of the columns), apply the fused
//               epilogue, store to global memory, release the accumulator.
// Two grouping modes:
//   M-grouped   rows of expert e are [off_e, off_e + n_e) of A and of the output; B is
//               the expert's own [K, N] (or [N, K]) slice. Tiles never straddle two
//               experts in the output: rows past n_e are computed but not stored.
//               (The library runs its M-grouped GEMMs on CTA pairs, in
//               grouped_gemm_pair_sm100.cuh, which reuses the epilogues below.)
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
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;                                   // bf16: 128 bytes of K per row
constexpr int kStages = 4;
constexpr int kThreads = 384;                          // 4 control warps + 8 epilogue warps
constexpr int kABytes = BM * BK * 2;                     // 16 KB
constexpr int kBBytes = BN * BK * 2;                     // 32 KB
constexpr int kChunkBytes = 64 * BK * 2;                 // one 64-wide MN chunk, 8 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kMaxE = 1024;
constexpr int kTmemCols = 512;                           // two 256-column accumulators
constexpr int kSmemBytes = 1024 /*align slack*/ + kStages * kStageBytes + 1024 /*barriers*/ +
                           3 * (kMaxE + 1) * 4 /*expert prefix tables, expert order*/;
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
  uint64_t timeout_ns;
};

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
      ti.m_blk = local % mt;
      ti.n_blk = local / mt;
      ti.row0 = row_off[ti.e] + ti.m_blk * TBM;
      ti.rows = min(TBM, n_e - ti.m_blk * TBM);
      ti.num_kb = K / gg::BK;
    }
    return ti;
  }
};

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

// Column of the B operand (output column space) of 64-wide chunk c of an N tile.
template <int EPI>
__device__ __forceinline__ int b_chunk_col(int n_blk, int c, int F) {
  if (EPI == EPI_SWIGLU) {
    const int n0 = n_blk * 128;
    return (c < 2) ? n0 + 64 * c : F + n0 + 64 * (c - 2);
  }
  return n_blk * gg::BN + 64 * c;
}

// Drain one BF16 accumulator tile: this thread owns row `tile_row` of the tile (its TMEM
// lane is folded into t_row) and the columns of `half`; applies the fused epilogue EPI.
template <int EPI>
__device__ __forceinline__ void bf16_epilogue_tile(const GemmParams& p, const TileInfo& ti, uint32_t t_row, int half,
                                                   int tile_row, int tile_bm) {
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
        if (EPI == EPI_STORE && p.out_f32) {
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
    const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(p.aux);
    __nv_bfloat16* dh = reinterpret_cast<__nv_bfloat16*>(p.out2);
    const int n0 = ti.n_blk * gg::BN;
    float dp = 0.f;
#pragma unroll 1
    for (int c0 = half * (gg::BN / 2); c0 < (half + 1) * (gg::BN / 2); c0 += 32) {
      // 32 columns per round: the saved h of the round is requested first, so its global
      // latency overlaps the two tensor-memory loads and their wait
      uint4 gva[4], uva[4];
      const bool cols_ok0 = row_ok && n0 + c0 < p.N;
      const bool cols_ok1 = row_ok && n0 + c0 + 16 < p.N;
      if (cols_ok0) {
        const uint4* gp = reinterpret_cast<const uint4*>(h + row * p.ld_aux + n0 + c0);
        const uint4* up = reinterpret_cast<const uint4*>(h + row * p.ld_aux + p.F + n0 + c0);
        gva[0] = gp[0];
        gva[1] = gp[1];
        uva[0] = up[0];
        uva[1] = up[1];
        if (cols_ok1) {
          gva[2] = gp[2];
          gva[3] = gp[3];
          uva[2] = up[2];
          uva[3] = up[3];
        }
      }
      uint32_t vv[2][16];
      tmem_ld_32x32b_x16(t_row + c0, vv[0]);
      tmem_ld_32x32b_x16(t_row + c0 + 16, vv[1]);
      tmem_wait_ld();
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int c = c0 + 16 * jj;
        const uint32_t* v = vv[jj];
        if (jj == 0 ? cols_ok0 : cols_ok1) {
          const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(gva + 2 * jj);
          const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(uva + 2 * jj);
          uint4 og[2], ou[2];
          uint32_t* ogw = reinterpret_cast<uint32_t*>(og);
          uint32_t* ouw = reinterpret_cast<uint32_t*>(ou);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float2 gg2 = __bfloat1622float2(g2[i]);
            const float2 uu2 = __bfloat1622float2(u2[i]);
            float dg[2], du[2];
            const float gs[2] = {gg2.x, gg2.y}, us[2] = {uu2.x, uu2.y};
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const float da = __uint_as_float(v[2 * i + j]);
              const float sg = 1.0f / (1.0f + expf(-gs[j]));
              const float sl = gs[j] * sg;
              dg[j] = da * pr * us[j] * (sg * (1.0f + gs[j] * (1.0f - sg)));
              du[j] = da * pr * sl;
              dp = fmaf(da, sl * us[j], dp);
            }
            ogw[i] = pack_bf16x2(dg[0], dg[1]);
            ouw[i] = pack_bf16x2(du[0], du[1]);
          }
          uint4* dg_dst = reinterpret_cast<uint4*>(dh + row * p.ldo2 + n0 + c);
          dg_dst[0] = og[0];
          dg_dst[1] = og[1];
          uint4* du_dst = reinterpret_cast<uint4*>(dh + row * p.ldo2 + p.F + n0 + c);
          du_dst[0] = ou[0];
          du_dst[1] = ou[1];
        }
      }
    }
    if (row_ok) p.dprob_part[(long long)(2 * ti.n_blk + half) * p.M + row] = dp;
  }
}

template <bool A_MN, bool B_MN, bool KGROUP, int EPI>
__global__ void __launch_bounds__(gg::kThreads, 1)
    grouped_gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const GemmParams p) {
  using namespace gg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* tfull = bars + 2 * kStages;
  uint64_t* tempty = bars + 2 * kStages + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* row_off = reinterpret_cast<int32_t*>(smem + kStages * kStageBytes + 1024);
  int32_t* tile_off = row_off + (kMaxE + 1);
  int32_t* order = tile_off + (kMaxE + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;

  // output tiling
  const int NT = (EPI == EPI_SWIGLU) ? (p.N / 128) : (p.N + BN - 1) / BN;
  const int MT = KGROUP ? (p.M + BM - 1) / BM : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 256);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  // expert prefix tables (warp 3): rows and tiles
  if (warp == 3) {
    int carry_r = 0, carry_t = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int n = (e < E) ? p.split_sizes[e] : 0;
      const int tiles = (e < E) ? (KGROUP ? MT * NT : ((n + BM - 1) / BM) * NT) : 0;
      int ir = n, it = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yr = __shfl_up_sync(0xffffffffu, ir, o);
        const int yt = __shfl_up_sync(0xffffffffu, it, o);
        if (lane >= o) {
          ir += yr;
          it += yt;
        }
      }
      if (e < E) {
        row_off[e] = carry_r + ir - n;
        tile_off[e] = carry_t + it - tiles;
      }
      carry_r += __shfl_sync(0xffffffffu, ir, 31);
      carry_t += __shfl_sync(0xffffffffu, it, 31);
    }
    if (lane == 0) {
      row_off[E] = carry_r;
      tile_off[E] = carry_t;
    }
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (KGROUP) {
    rank_experts_by_rows(row_off, E, order);
    __syncthreads();
  }

  TileWalker<KGROUP> walk{row_off, tile_off, E, MT, NT, p.K, order};
  const int total = walk.total();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const TileInfo ti = walk.decode(t);
        for (int kb = 0; kb < ti.num_kb; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          uint8_t* a_dst = sA + stage * kABytes;
          uint8_t* b_dst = sB + stage * kBBytes;
          const int k0 = kb * BK;
          if (!A_MN) {
            tma_load_3d(a_dst, &tmA, &full[stage], k0, ti.row0, 0);
          } else if (KGROUP) {
            // both 64-column chunks in one copy (chunked view, box {64, 64 k rows, 2, 1})
            tma_load_4d(a_dst, &tmA, &full[stage], 0, ti.row0 + k0, ti.m_blk * (BM / 64), 0);
          } else {
#pragma unroll
            for (int c = 0; c < 2; ++c)
              tma_load_3d(a_dst + c * kChunkBytes, &tmA, &full[stage], ti.m_blk * BM + 64 * c, ti.row0 + k0, 0);
          }
          if (!B_MN) {
            tma_load_3d(b_dst, &tmB, &full[stage], k0, ti.n_blk * BN, ti.e);
          } else if (KGROUP) {
            // all four 64-column chunks in one copy (box {64, 64 k rows, 4, 1})
            tma_load_4d(b_dst, &tmB, &full[stage], 0, ti.row0 + k0, ti.n_blk * (BN / 64), 0);
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              tma_load_3d(b_dst + c * kChunkBytes, &tmB, &full[stage], b_chunk_col<EPI>(ti.n_blk, c, p.F), k0, ti.e);
          }
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        // drain: let the copies already issued land before the CTA can exit
        int st = stage, ph = phase;
        for (int i = 0; i < min(issued, kStages); ++i) {
          if (--st < 0) {
            st = kStages - 1;
            ph ^= 1;
          }
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(&full[st], ph) && global_timer_ns() - t0 < 100000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = make_idesc_bf16(BM, BN, A_MN, B_MN);
    int stage = 0;
    uint32_t phase = 0;
    int lt = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++lt) {
      const TileInfo ti = walk.decode(t);
      const int acc = lt & 1;
      const uint32_t acc_phase = (lt >> 1) & 1;
      if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, p.timeout_ns)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      for (int kb = 0; kb < ti.num_kb; ++kb) {
        if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        int ksteps = BK / 16;   // K=16 MMAs of this stage
        if (KGROUP && (kb + 1) * BK > ti.rows) {
          // clip the contraction at the end of the expert's rows: MMAs only over the
          // expert's K-rows; inside the last, partial 16-row step zero the rows >= valid
          // of all six 64-wide operand chunks (A 2, B 4; row r of a chunk at r * 128 bytes)
          const int valid = ti.rows - kb * BK;
          ksteps = (valid + 15) / 16;
          const int zr = ksteps * 16 - valid;   // 0..15 rows
          if (zr > 0) {
            uint8_t* a_st = sA + stage * kABytes;
            uint8_t* b_st = sB + stage * kBBytes;
            for (int i = lane; i < 6 * zr * 8; i += 32) {
              const int v = i & 7, rc = i >> 3;
              const int c = rc / zr, r = rc - c * zr;
              uint8_t* base = (c < 2) ? a_st + c * kChunkBytes : b_st + (c - 2) * kChunkBytes;
              *reinterpret_cast<uint4*>(base + (valid + r) * 128 + v * 16) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
          }
          __syncwarp();
        }
        if (lane == 0) {
          const uint32_t a_addr = smem_u32(sA + stage * kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * kBBytes);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            if (kk >= ksteps) break;
            const uint64_t adesc = A_MN ? make_sdesc(a_addr + kk * 2048, kChunkBytes, 1024, 2)
                                        : make_sdesc(a_addr + kk * 32, 16, 1024, 2);
            const uint64_t bdesc = B_MN ? make_sdesc(b_addr + kk * 2048, kChunkBytes, 1024, 2)
                                        : make_sdesc(b_addr + kk * 32, 16, 1024, 2);
            mma_bf16_ss(d_tmem, adesc, bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      if (lane == 0) {
        if (ti.num_kb > 0)
          mma_commit(&tfull[acc]);
        else
          mbar_arrive(&tfull[acc]);
      }
      __syncwarp();
    }
  } else if (warp >= 4) {
    // ----------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int half = (warp - 4) >> 2;       // which half of the tile's columns it drains
    const int r_local = q * 32 + lane;      // accumulator row owned by this thread
    int lt = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++lt) {
      const TileInfo ti = walk.decode(t);
      const int acc = lt & 1;
      const uint32_t acc_phase = (lt >> 1) & 1;
      if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, p.timeout_ns)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + acc * BN + ((uint32_t)(q * 32) << 16);
      bf16_epilogue_tile<EPI>(p, ti, t_row, half, r_local, BM);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
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
