// Token-side kernels of the MoE expert-MLP path: top-k router softmax, the stable
// expert-contiguous permutation (index build + data movement, with an optional fused
// MXFP8 row quantisation), the unpermute/combine, and the standalone MXFP8 quantiser.
//
// Pages: "Efficient MoE training for biological foundation models" (sitech.ge section
// "Grouped experts instead of a Python loop"; news.bpdata.com sections 1-2): tokens are
// routed to a few experts, grouped per expert with per-expert counts (split_sizes), and
// MXFP8 keeps one scale per 32 consecutive values.
#pragma once
#include <cuda_fp8.h>

#include "ptx_sm100.cuh"

namespace moe {

constexpr int kPermuteChunk = 1024;   // slots per block in the index build
constexpr int kPermuteThreads = 256;  // 8 warps, 128 consecutive slots per warp
constexpr int kMaxExperts = 1024;

// ------------------------------------------------------------------------ routing
// One warp routes one token: softmax over all E logits in fp32, then the k largest
// logits (ties -> lower expert index) in descending order; with renorm the k
// probabilities are divided by their sum. Lane j (< k) returns choice j.
template <int VPL>  // logits held per lane: ceil(E / 32)
__device__ __forceinline__ void route_one_token(const float* __restrict__ row, int E, int k, int renorm, int lane,
                                                int& e_out, float& p_out) {
  float v[VPL];
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? row[e] : -INFINITY;
    m = fmaxf(m, v[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i)
    if (lane + 32 * i < E) s += expf(v[i] - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);

  uint32_t taken = 0;
  float psum = 0.f;
  float pk = 0.f;   // lane j (< k) keeps probability j
  int ek = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    const float p = expf(bv - m) / s;
    psum += p;
    if (lane == j) {
      pk = p;
      ek = be;
    }
  }
  e_out = ek;
  p_out = renorm ? pk / psum : pk;
}

// The same routing with W lanes per token (E <= W <= 32, W a power of two), so that a
// warp routes 32 / W tokens at once; lane `sub` of its group holds logit v of expert sub
// (-inf past E). The results are those of route_one_token bit for bit: there, lanes past
// E enter the max, sum and arg-max trees as -inf, exact zeros and (-inf, no expert) and
// change nothing, and the trees over the first W lanes use the same xor steps.
template <int W>
__device__ __forceinline__ void route_one_token_narrow(float v, int E, int k, int renorm, int sub, int& e_out,
                                                       float& p_out) {
  float m = v;
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o, W));
  float s = (sub < E) ? expf(v - m) : 0.f;
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o, W);
  bool taken = false;
  float psum = 0.f, pk = 0.f;
  int ek = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
    if (sub < E && !taken && (v > bv || (v == bv && sub < be))) {
      bv = v;
      be = sub;
    }
#pragma unroll
    for (int o = W / 2; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o, W);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o, W);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if (be == sub) taken = true;
    const float p = expf(bv - m) / s;
    psum += p;
    if (sub == j) {
      pk = p;
      ek = be;
    }
  }
  e_out = ek;
  p_out = renorm ? pk / psum : pk;
}

template <int VPL>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                         int renorm, int32_t* __restrict__ idx,
                                                         float* __restrict__ prob) {
  const int lane = threadIdx.x & 31;
  const int warps_per_block = blockDim.x >> 5;
  for (int t = blockIdx.x * warps_per_block + (threadIdx.x >> 5); t < T; t += gridDim.x * warps_per_block) {
    int e;
    float p;
    route_one_token<VPL>(logits + (size_t)t * E, E, k, renorm, lane, e, p);
    if (lane < k) {
      idx[(size_t)t * k + lane] = e;
      prob[(size_t)t * k + lane] = p;
    }
  }
}

// Router backward, one warp per token: dlogits [T, E] from dL/dprob [T, k] and the
// forward's idx / prob. The forward is s = softmax(l), q_j = s[idx_j], p_j = q_j / Z with
// Z = sum_j q_j (renorm) or p_j = q_j. By the chain rule dl_b = s_b (ds_b - <ds, s>) with
// ds_b the sum of dq_j over the slots that chose b.
//  * renorm: dq_j = (dprob_j - D) / Z with D = sum_m dprob_m p_m; then <ds, s> = 0 and
//    s_b ds_b = p_j (dprob_j - D), so dl_b = sum over slots j choosing b of p_j (dprob_j - D)
//    and 0 for experts nobody chose; the logits are not needed.
//  * no renorm: dq_j = dprob_j and s is recomputed from the logits in fp32.
template <int VPL>
__global__ void __launch_bounds__(256) route_bwd_kernel(const float* __restrict__ logits,
                                                        const int32_t* __restrict__ idx,
                                                        const float* __restrict__ prob,
                                                        const float* __restrict__ dprob, int T, int E, int k,
                                                        int renorm, float* __restrict__ dlogits) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
    int ej = -1;
    float pj = 0.f, dj = 0.f;
    if (lane < k) {
      ej = idx[(size_t)t * k + lane];
      pj = prob[(size_t)t * k + lane];
      dj = dprob[(size_t)t * k + lane];
      if (ej < 0 || ej >= E) {
        flag_error(DEVERR_BAD_INDEX);
        ej = -1;
      }
    }
    float acc[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
    float* out = dlogits + (size_t)t * E;
    if (renorm) {
      float D = dj * pj;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) D += __shfl_xor_sync(0xffffffffu, D, o);
      const float gj = pj * (dj - D);
      for (int j = 0; j < k; ++j) {
        const int eb = __shfl_sync(0xffffffffu, ej, j);
        const float gb = __shfl_sync(0xffffffffu, gj, j);
#pragma unroll
        for (int i = 0; i < VPL; ++i)
          if (lane + 32 * i == eb) acc[i] += gb;
      }
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (lane + 32 * i < E) out[lane + 32 * i] = acc[i];
    } else {
      // ds_b: sum of dprob_j over the slots that chose b
      for (int j = 0; j < k; ++j) {
        const int eb = __shfl_sync(0xffffffffu, ej, j);
        const float db = __shfl_sync(0xffffffffu, dj, j);
#pragma unroll
        for (int i = 0; i < VPL; ++i)
          if (lane + 32 * i == eb) acc[i] += db;
      }
      const float* row = logits + (size_t)t * E;
      float v[VPL];
      float m = -INFINITY;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int e = lane + 32 * i;
        v[i] = (e < E) ? row[e] : -INFINITY;
        m = fmaxf(m, v[i]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float z = 0.f;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        v[i] = (lane + 32 * i < E) ? expf(v[i] - m) : 0.f;
        z += v[i];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      const float inv = 1.0f / z;
      float dot = 0.f;   // <ds, s>
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        v[i] *= inv;
        dot = fmaf(acc[i], v[i], dot);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        if (lane + 32 * i < E) out[lane + 32 * i] = v[i] * (acc[i] - dot);
    }
  }
}

// ------------------------------------------------------------- permutation index
// Pass 1: per-block expert histogram of a chunk of kPermuteChunk consecutive slots.
__global__ void __launch_bounds__(kPermuteThreads) permute_hist_kernel(const int32_t* __restrict__ idx, int R,
                                                                       int E, int32_t* __restrict__ counts) {
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int s0 = blockIdx.x * kPermuteChunk;
  for (int i = threadIdx.x; i < kPermuteChunk; i += blockDim.x) {
    const int s = s0 + i;
    if (s < R) {
      const int e = idx[s];
      if (e >= 0 && e < E)
        atomicAdd(&hist[e], 1);
      else
        flag_error(DEVERR_BAD_INDEX);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) counts[(size_t)blockIdx.x * E + e] = hist[e];
}

// Pass 2 (one block of 1024 threads, E <= 1024): split_sizes, offsets, and the first
// row of every (block, expert) pair, written over the counts. Threads form a [P][E]
// grid (P = 1024 / E) that splits the blocks into P contiguous ranges. `sm` holds
// (P + 1) * E int32. The counts are read past L1 (they may come from other SMs).
__device__ __forceinline__ void scan_block_counts(int32_t* __restrict__ counts, int nblk, int E, int R,
                                                  int32_t* __restrict__ split_sizes, int32_t* __restrict__ offsets,
                                                  int32_t* sm, int32_t* wsum) {
  const int P = max(1, (int)blockDim.x / E);
  int32_t* part = sm;          // [P][E] partial sums, then their exclusive prefix over p
  int32_t* off = sm + P * E;   // [E] first row of each expert
  const int per = (nblk + P - 1) / P;
  for (int tid = threadIdx.x; tid < E * P; tid += blockDim.x) {
    const int p = tid / E, e = tid % E;
    int acc = 0;
    for (int b = p * per; b < min(nblk, (p + 1) * per); ++b) acc += __ldcg(counts + (size_t)b * E + e);
    part[p * E + e] = acc;
  }
  __syncthreads();
  const int e = threadIdx.x;
  int tot = 0;
  if (e < E) {
    for (int p = 0; p < P; ++p) {
      const int c = part[p * E + e];
      part[p * E + e] = tot;
      tot += c;
    }
    split_sizes[e] = tot;
  }
  // block-wide exclusive scan of tot over e
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < (int)(blockDim.x >> 5)) ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    wsum[lane] = w;   // inclusive over warps
  }
  __syncthreads();
  const int excl = incl - tot + (warp > 0 ? wsum[warp - 1] : 0);
  if (e < E) {
    off[e] = excl;
    offsets[e] = excl;
    if (e == E - 1) {
      offsets[E] = excl + tot;
      if (excl + tot != R) flag_error(DEVERR_SPLIT_SUM);
    }
  }
  __syncthreads();
  for (int tid = threadIdx.x; tid < E * P; tid += blockDim.x) {
    const int p = tid / E, ee = tid % E;
    int base = off[ee] + part[p * E + ee];
    for (int b = p * per; b < min(nblk, (p + 1) * per); ++b) {
      const int c = __ldcg(counts + (size_t)b * E + ee);
      counts[(size_t)b * E + ee] = base;
      base += c;
    }
  }
}

__global__ void __launch_bounds__(1024) permute_scan_kernel(int32_t* __restrict__ counts, int nblk, int E, int R,
                                                            int32_t* __restrict__ split_sizes,
                                                            int32_t* __restrict__ offsets) {
  extern __shared__ int32_t sm[];
  __shared__ int32_t wsum[32];
  scan_block_counts(counts, nblk, E, R, split_sizes, offsets, sm, wsum);
}

// Route + index build in one launch (1024 threads per block, k divides kPermuteChunk):
// block b routes tokens [b * 1024/k, (b+1) * 1024/k) — exactly the slots of histogram
// chunk b — and writes that chunk's expert histogram; the last block to finish (a
// device-wide counter, zeroed before the launch and reset by that block) then runs the
// scan of pass 2. Replaces the route, histogram and scan launches of the unfused path.
// W < 32 (E <= W, VPL = 1): W lanes per token, 32 / W tokens per warp at a time (every
// block routes its 1024/k tokens whatever T is, so its latency sets the launch's).
template <int VPL, int W = 32>
__global__ void __launch_bounds__(1024, 1) route_index_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                              int renorm, int32_t* __restrict__ idx,
                                                              float* __restrict__ prob, int32_t* __restrict__ counts,
                                                              int nblk, int32_t* __restrict__ split_sizes,
                                                              int32_t* __restrict__ offsets,
                                                              unsigned int* __restrict__ done) {
  extern __shared__ int32_t sm[];       // hist [E], then the scan's (P + 1) * E
  __shared__ int32_t wsum[32];
  __shared__ int is_last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tpb = kPermuteChunk / k;
  const int t0 = blockIdx.x * tpb, t1 = min(T, t0 + tpb);
  for (int e = threadIdx.x; e < E; e += blockDim.x) sm[e] = 0;
  __syncthreads();
  if (W < 32) {
    constexpr int G = 32 / W;   // tokens per warp at a time
    const int sub = lane % W, grp = lane / W;
    const int step = (int)(blockDim.x >> 5) * G;
    auto load = [&](int t) { return (t < t1 && sub < E) ? __ldg(logits + (size_t)t * E + sub) : -INFINITY; };
    float vn = load(t0 + warp * G + grp);   // the next tokens' logits are loaded a round ahead
    for (int tb = t0 + warp * G; tb < t1; tb += step) {   // warp-uniform bound
      const int t = tb + grp;
      const bool ok = t < t1;
      const float v = vn;
      vn = load(t + step);
      int e;
      float p;
      route_one_token_narrow<W>(v, E, k, renorm, sub, e, p);
      if (ok && sub < k) {
        idx[(size_t)t * k + sub] = e;
        prob[(size_t)t * k + sub] = p;
        atomicAdd(&sm[e], 1);
      }
    }
  } else {
    for (int t = t0 + warp; t < t1; t += (int)(blockDim.x >> 5)) {
      int e;
      float p;
      route_one_token<VPL>(logits + (size_t)t * E, E, k, renorm, lane, e, p);
      if (lane < k) {
        idx[(size_t)t * k + lane] = e;
        prob[(size_t)t * k + lane] = p;
        atomicAdd(&sm[e], 1);
      }
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) counts[(size_t)blockIdx.x * E + e] = sm[e];
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(done, 1u) == (unsigned)(nblk - 1));
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  scan_block_counts(counts, nblk, E, T * k, split_sizes, offsets, sm, wsum);
  if (threadIdx.x == 0) *done = 0u;
}

// Pass 3: stable ranks inside the block. Warp w owns slots [w*128, w*128+128) of the
// chunk; ranks follow slot order: earlier warps, then earlier lanes/iterations.
__global__ void __launch_bounds__(kPermuteThreads) permute_rowmap_kernel(const int32_t* __restrict__ idx,
                                                                         const float* __restrict__ prob, int R,
                                                                         int E, const int32_t* __restrict__ base,
                                                                         int32_t* __restrict__ row_map,
                                                                         float* __restrict__ probs_perm) {
  constexpr int kWarps = kPermuteThreads / 32;
  constexpr int kPerWarp = kPermuteChunk / kWarps;   // 128
  extern __shared__ int32_t cnt[];                   // [kWarps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  const int s_warp = blockIdx.x * kPermuteChunk + warp * kPerWarp;
  const unsigned lt = (1u << lane) - 1u;
  // count this warp's slots per expert
  for (int it = 0; it < kPerWarp; it += 32) {
    const int s = s_warp + it + lane;
    int e = (s < R) ? idx[s] : -1;
    if (e >= E) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && (peers & lt) == 0) cnt[warp * E + e] += __popc(peers);
  }
  __syncthreads();
  // exclusive prefix across warps, seeded with the block's starting row per expert
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = base[(size_t)blockIdx.x * E + e];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int c = cnt[w * E + e];
      cnt[w * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  for (int it = 0; it < kPerWarp; it += 32) {
    const int s = s_warp + it + lane;
    int e = (s < R) ? idx[s] : -1;
    if (e >= E) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0) {
      const int row = cnt[warp * E + e] + __popc(peers & lt);
      row_map[s] = row;
      if (probs_perm) probs_perm[row] = prob[s];
    } else if (s < R) {
      row_map[s] = -1;
    }
    __syncwarp();
    if (e >= 0 && (peers & lt) == 0) cnt[warp * E + e] += __popc(peers);
    __syncwarp();
  }
}

// Capacity-padded dispatch: slot s of expert e, ranked `rank` among that expert's slots in
// slot order (the stable permutation's row minus the expert's offset), goes to row
// e * C + rank of the padded [E * C] layout if rank < C, else it is dropped (row -1).
// Threads e < E also write the padded layout's split sizes (all C), offsets and the
// number of slots each expert kept.
__global__ void __launch_bounds__(256) capacity_rows_kernel(const int32_t* __restrict__ idx,
                                                            const int32_t* __restrict__ row_map_full,
                                                            const int32_t* __restrict__ split_full,
                                                            const int32_t* __restrict__ offsets_full,
                                                            const float* __restrict__ prob, int R, int E, int C,
                                                            int32_t* __restrict__ row_map, float* __restrict__ probs_perm,
                                                            int32_t* __restrict__ split_sizes,
                                                            int32_t* __restrict__ offsets, int32_t* __restrict__ kept) {
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  for (int s = tid; s < R; s += gridDim.x * blockDim.x) {
    const int e = idx[s];
    const int r = row_map_full[s];
    if (e < 0 || e >= E || r < 0) {
      row_map[s] = -1;
      continue;
    }
    const int rank = r - offsets_full[e];
    if (rank < C) {
      const int row = e * C + rank;
      row_map[s] = row;
      if (probs_perm) probs_perm[row] = prob[s];
    } else {
      row_map[s] = -1;
    }
  }
  if (tid < E) {
    split_sizes[tid] = C;
    offsets[tid] = tid * C;
    if (kept) kept[tid] = min(split_full[tid], C);
    if (tid == E - 1) offsets[E] = E * C;
  }
}

// ------------------------------------------------------------- per-tensor FP8
// Current scaling: one scale per tensor (a batch of tensors: one per blockIdx.y), s =
// fmt_max / max |x| in fp32 (1 for an all-zero tensor), codes = the fp32 product x * s
// rounded to E4M3 or E5M2 (nearest even, saturating).
__device__ __forceinline__ float fp8_max(int e5m2) { return e5m2 ? 57344.0f : 448.0f; }

// max |x| of each tensor (n8 groups of 8 bf16 per tensor) into amax_bits[b] (fp32 bits;
// zero before the launch).
__global__ void __launch_bounds__(256) amax_bf16_kernel(const uint4* __restrict__ in, long long n8,
                                                        unsigned int* __restrict__ amax_bits) {
  const uint4* src = in + (long long)blockIdx.y * n8;
  float m = 0.f;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    const uint4 v = __ldg(src + i);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(h[j]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  const unsigned int r = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
  if ((threadIdx.x & 31) == 0 && r) atomicMax(amax_bits + blockIdx.y, r);
}

// scale[b] = fmt_max / amax[b] in fp32 (1 when amax is 0).
__global__ void fp8_scale_kernel(const unsigned int* __restrict__ amax_bits, int batch, int e5m2,
                                 float* __restrict__ scale) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < batch; b += gridDim.x * blockDim.x) {
    const float a = __uint_as_float(amax_bits[b]);
    scale[b] = a > 0.f ? fp8_max(e5m2) / a : 1.0f;
  }
}

__device__ __forceinline__ uint32_t fp8_pack4(float a, float b, float c, float d, int e5m2) {
  const __nv_fp8_interpretation_t f = e5m2 ? __NV_E5M2 : __NV_E4M3;
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, f) |
         ((uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, f) << 16);
}

// codes of each tensor (n8 groups of 8 per tensor, blockIdx.y = tensor) with its scale.
__global__ void __launch_bounds__(256) fp8_cast_kernel(const uint4* __restrict__ in, long long n8,
                                                       const float* __restrict__ scale, int e5m2,
                                                       uint2* __restrict__ codes) {
  const uint4* src = in + (long long)blockIdx.y * n8;
  uint2* dst = codes + (long long)blockIdx.y * n8;
  const float s = scale[blockIdx.y];
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    const uint4 v = __ldg(src + i);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
    float f[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 p = __bfloat1622float2(h[j]);
      f[2 * j] = p.x * s;
      f[2 * j + 1] = p.y * s;
    }
    dst[i] = make_uint2(fp8_pack4(f[0], f[1], f[2], f[3], e5m2), fp8_pack4(f[4], f[5], f[6], f[7], e5m2));
  }
}

// The same with the output transposed: in [b][rows][cols] -> codes [b][cols][rows]
// (rows, cols multiples of 32). A block moves a 32 x 32 tile through shared memory.
__global__ void __launch_bounds__(256) fp8_cast_transpose_kernel(const __nv_bfloat16* __restrict__ in, int rows,
                                                                 int cols, const float* __restrict__ scale, int e5m2,
                                                                 uint8_t* __restrict__ codes) {
  __shared__ float tile[32][33];
  const int b = blockIdx.z;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  const float s = scale[b];
  const __nv_bfloat16* src = in + (size_t)b * rows * cols;
  uint8_t* dst = codes + (size_t)b * rows * cols;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8 threads
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty + 8 * i;
    tile[r][tx] = __bfloat162float(src[(size_t)(r0 + r) * cols + c0 + tx]) * s;
  }
  __syncthreads();
  // thread (ty, tx/4...): each of the 256 threads writes 4 consecutive codes of one output row
  const int orow = threadIdx.x >> 3, oc = (threadIdx.x & 7) * 4;   // output row = input column
  const uint32_t w = fp8_pack4(tile[oc][orow], tile[oc + 1][orow], tile[oc + 2][orow], tile[oc + 3][orow], e5m2);
  *reinterpret_cast<uint32_t*>(dst + (size_t)(c0 + orow) * rows + r0 + oc) = w;
}

// ------------------------------------------------------------ permutation data
// xp[row_map[t*k + j]] = x[t] for j < k. One warp per token, 16-byte vectors.
__global__ void __launch_bounds__(256) permute_rows_bf16_kernel(const uint4* __restrict__ x, int T, int H8, int k,
                                                                const int32_t* __restrict__ row_map,
                                                                uint4* __restrict__ xp) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
    int rows[8];
    const int kk = min(k, 8);
    for (int j = 0; j < kk; ++j) rows[j] = row_map[(size_t)t * k + j];
    const uint4* src = x + (size_t)t * H8;
    for (int c = lane; c < H8; c += 32) {
      const uint4 v = __ldg(src + c);
      for (int j = 0; j < kk; ++j)
        if (rows[j] >= 0) xp[(size_t)rows[j] * H8 + c] = v;
    }
    for (int j = 8; j < k; ++j) {   // k > 8: rare, plain loop
      const int r = row_map[(size_t)t * k + j];
      if (r < 0) continue;
      for (int c = lane; c < H8; c += 32) xp[(size_t)r * H8 + c] = __ldg(src + c);
    }
  }
}

// Quantise 8 consecutive bf16 values held by one lane of a 4-lane group (one 32-value
// block per group): amax over the group, E8M0 code = max(biased_exp(amax) - 8, 0),
// elements scaled by 2^(127 - code) (exact) and converted with round-to-nearest-even,
// saturating to +-448.
__device__ __forceinline__ uint2 mxfp8_quant8(const uint4 v, uint8_t* scale_out) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
  float f[8];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 p = __bfloat1622float2(h[i]);
    f[2 * i] = p.x;
    f[2 * i + 1] = p.y;
    amax = fmaxf(amax, fmaxf(fabsf(p.x), fabsf(p.y)));
  }
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  const int bexp = (int)((__float_as_uint(amax) >> 23) & 0xFF);
  const int code = max(bexp - 8, 0);
  *scale_out = (uint8_t)code;
  const float inv = __uint_as_float((uint32_t)(254 - code) << 23);   // 2^(127 - code)
  uint32_t w[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const __nv_fp8x2_storage_t lo =
        __nv_cvt_float2_to_fp8x2(make_float2(f[4 * i] * inv, f[4 * i + 1] * inv), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi =
        __nv_cvt_float2_to_fp8x2(make_float2(f[4 * i + 2] * inv, f[4 * i + 3] * inv), __NV_SATFINITE, __NV_E4M3);
    w[i] = (uint32_t)lo | ((uint32_t)hi << 16);
  }
  return make_uint2(w[0], w[1]);
}

// MXFP8 permute: quantise each token row along H once, write codes/scales to its k rows.
// Every lane of a warp runs the same number of iterations (the 4-lane shuffles inside
// the quantiser need the whole warp); lanes past the row end work on zeros.
__global__ void __launch_bounds__(256) permute_rows_mxfp8_kernel(const uint4* __restrict__ x, int T, int H, int k,
                                                                 const int32_t* __restrict__ row_map,
                                                                 uint8_t* __restrict__ xq,
                                                                 uint8_t* __restrict__ xs) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int H8 = H >> 3;
  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
    const uint4* src = x + (size_t)t * H8;
    for (int c0 = 0; c0 < H8; c0 += 32) {
      const int c = c0 + lane;
      const bool live = c < H8;   // H8 is a multiple of 4: a 4-lane group is all live or all dead
      uint8_t sc;
      const uint2 q = mxfp8_quant8(live ? __ldg(src + c) : make_uint4(0, 0, 0, 0), &sc);
      if (!live) continue;
      for (int j = 0; j < k; ++j) {
        const int r = row_map[(size_t)t * k + j];
        if (r < 0) continue;
        *reinterpret_cast<uint2*>(xq + (size_t)r * H + (size_t)c * 8) = q;
        if ((lane & 3) == 0) xs[(size_t)r * (H >> 5) + (c >> 2)] = sc;
      }
    }
  }
}

// ------------------------------------------------------------- unpermute/combine
// row_token[row_map[s]] = s / k: the token of every permuted row (for the fused combine).
__global__ void __launch_bounds__(256) row_token_kernel(const int32_t* __restrict__ row_map, int R, int k,
                                                        int32_t* __restrict__ row_token) {
  for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < R; s += gridDim.x * blockDim.x) {
    const int r = row_map[s];
    if (r >= 0 && r < R)
      row_token[r] = s / k;
    else
      flag_error(DEVERR_BAD_INDEX);
  }
}

// out[i] = bf16(in[i]) for n8 groups of 8 fp32 values (the fused combine's last step).
__global__ void __launch_bounds__(256) f32_to_bf16_kernel(const float4* __restrict__ in, long long n8,
                                                          uint4* __restrict__ out) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
    const float4 a = in[2 * i], b = in[2 * i + 1];
    out[i] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
  }
}

// out[t] = sum_j w_tj * yp[row_map[t*k+j]] (w = 1 without prob), fp32 accumulation in
// slot order, rounded once to bf16.
__global__ void __launch_bounds__(256) unpermute_bf16_kernel(const uint4* __restrict__ yp,
                                                             const int32_t* __restrict__ row_map,
                                                             const float* __restrict__ prob, int T, int H8, int k,
                                                             uint4* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < T; t += gridDim.x * wpb) {
    for (int c = lane; c < H8; c += 32) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int j = 0; j < k; ++j) {
        const int r = row_map[(size_t)t * k + j];
        if (r < 0) continue;
        const float w = prob ? prob[(size_t)t * k + j] : 1.0f;
        const uint4 v = __ldg(yp + (size_t)r * H8 + c);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 p = __bfloat1622float2(h[i]);
          acc[2 * i] = fmaf(w, p.x, acc[2 * i]);
          acc[2 * i + 1] = fmaf(w, p.y, acc[2 * i + 1]);
        }
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      out[(size_t)t * H8 + c] = o;
    }
  }
}

// dprob[t, j] = dprobs_perm[row_map[t*k + j]]
__global__ void gather_slots_f32_kernel(const float* __restrict__ src, const int32_t* __restrict__ row_map, int R,
                                        float* __restrict__ dst) {
  for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < R; s += gridDim.x * blockDim.x) {
    const int r = row_map[s];
    dst[s] = (r >= 0) ? src[r] : 0.f;
  }
}

// ------------------------------------------------------ MMA scale-atom layout
// The block-scaled MMA reads its scales from tensor memory, filled by tcgen05.cp from a
// 512-byte shared-memory atom per 128 rows x 4 k-blocks (4 x 32 K values): row r of the
// group is the 32-bit word (r % 32) * 4 + r / 32 and k-block kb its byte kb % 4. Keeping
// scales in global memory already arranged as these atoms lets a GEMM stage fetch its
// scales with one bulk copy per 128 rows. Atom (g, j) covers row group g and k-blocks
// [4j, 4j+4); atoms of one row group are consecutive: offset (g * KB4 + j) * 512.
__host__ __device__ __forceinline__ size_t mma_scale_offset(size_t group, int r, int kb, int kb4_per_row) {
  return ((group * (size_t)kb4_per_row + (size_t)(kb >> 2)) * 128 + (size_t)((r & 31) * 4 + (r >> 5))) * 4 +
         (size_t)(kb & 3);
}

// Plain [R, K/32] scales of expert-contiguous rows -> MMA atoms grouped per expert tile:
// row group g = (sum over e' < e of ceil(n_e' / 128)) + m for rows [off_e + 128 m, +128) of
// expert e; rows past the expert's end get zero scales. One thread per (group, row,
// 4-k-block word). Each block rebuilds the expert prefix tables from split_sizes.
__global__ void __launch_bounds__(256) scales_to_atoms_kernel(const uint8_t* __restrict__ plain,
                                                              const int32_t* __restrict__ split_sizes, int E, int KS,
                                                              long long max_groups, uint32_t* __restrict__ atoms) {
  extern __shared__ int32_t tabs[];   // [E+1] row offsets, [E+1] group offsets
  int32_t* roff = tabs;
  int32_t* goff = tabs + E + 1;
  if (threadIdx.x < 32) {   // warp prefix sums of split_sizes and of their 128-row groups
    const int lane = threadIdx.x;
    int cr = 0, cg = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int n = (e < E) ? split_sizes[e] : 0;
      const int gn = (n + 127) / 128;
      int ir = n, ig = gn;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yr = __shfl_up_sync(0xffffffffu, ir, o);
        const int yg = __shfl_up_sync(0xffffffffu, ig, o);
        if (lane >= o) {
          ir += yr;
          ig += yg;
        }
      }
      if (e < E) {
        roff[e] = cr + ir - n;
        goff[e] = cg + ig - gn;
      }
      cr += __shfl_sync(0xffffffffu, ir, 31);
      cg += __shfl_sync(0xffffffffu, ig, 31);
    }
    if (lane == 0) {
      roff[E] = cr;
      goff[E] = cg;
    }
  }
  __syncthreads();
  const int KB4 = KS / 4;
  const long long total = (long long)goff[E] * KB4 * 128;
  (void)max_groups;
  for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < total;
       w += (long long)gridDim.x * blockDim.x) {
    const int word = (int)(w % 128);
    const long long gj = w / 128;
    const int j = (int)(gj % KB4);
    const int g = (int)(gj / KB4);
    int lo = 0, hi = E - 1;   // expert whose groups contain g
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (goff[mid] <= g) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int r = (word & 3) * 32 + (word >> 2);   // inverse of (r % 32) * 4 + r / 32
    const int l = (g - goff[e]) * 128 + r;
    uint32_t v = 0;
    if (l < roff[e + 1] - roff[e]) v = *reinterpret_cast<const uint32_t*>(plain + (size_t)(roff[e] + l) * KS + 4 * j);
    atoms[w] = v;
  }
}

// ------------------------------------------------------------ MXFP8 quantiser
// E4M3 codes of 32 fp32 values (one lane's row) quantised along the 32 LANES of the warp:
// for each column j the block maximum is the warp-wide max of |v[j]| (one floating-point
// redux with the absolute-value modifier), E8M0 code max(exp(amax) - 8, 0), element
// scaled by 2^(127 - code) exactly and rounded to nearest even with saturation. Lanes
// that hold no row pass zeros. Every lane of the warp must call this together. Returns
// the codes in `w` (byte j = column j) and, in lane j, the scale code of column j.
// The scale factor's bits come straight from the maximum's exponent field e:
// (254 - max(e - 8, 0)) << 23 = min((262 - e) << 23, 254 << 23), unsigned. Lane j's own
// column maximum is picked from the 32 (warp-uniform) maxima by a select tree on the bits
// of j, built as the columns go (31 selects, not a compare and a select per column).
__device__ __forceinline__ uint32_t quant_cols_warp32(const float (&v)[32], uint32_t (&w)[8], int lane) {
  uint32_t lv[5];   // pending select-tree nodes, one per level
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const uint32_t m0 = warp_max_abs_bits(v[j]);
    const uint32_t m1 = warp_max_abs_bits(v[j + 1]);
    const float i0 = __uint_as_float(min(0x83000000u - (m0 & 0x7F800000u), 0x7F000000u));
    const float i1 = __uint_as_float(min(0x83000000u - (m1 & 0x7F800000u), 0x7F000000u));
    const uint32_t pair =
        (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(v[j] * i0, v[j + 1] * i1), __NV_SATFINITE, __NV_E4M3);
    if ((j & 2) == 0)
      w[j >> 2] = pair;
    else
      w[j >> 2] |= pair << 16;
    // the tree: node of pair i = j / 2 at level 0, merged upwards while i's low bits are 1
    uint32_t node = (lane & 1) ? m1 : m0;
    const int i = j >> 1;
#pragma unroll
    for (int l = 0; l < 4; ++l) {
      if (((i >> l) & 1) == 0) {
        lv[l] = node;
        break;
      }
      node = ((lane >> (l + 1)) & 1) ? node : lv[l];
    }
    if (i == 15) lv[4] = node;
  }
  return (uint32_t)max((int)(lv[4] >> 23) - 8, 0);
}

// E4M3 codes of 32 fp32 values of one row quantised as one block along the row; returns
// the block's scale code.
__device__ __forceinline__ uint32_t quant_row32(float (&v)[32], uint32_t (&w)[8]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int code = max((int)((__float_as_uint(amax) >> 23) & 0xFF) - 8, 0);
  const float inv = __uint_as_float((uint32_t)(254 - code) << 23);
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] *= inv;
  pack_e4m3x16(v, *reinterpret_cast<uint32_t(*)[4]>(&w[0]));
  pack_e4m3x16(v + 16, *reinterpret_cast<uint32_t(*)[4]>(&w[4]));
  return (uint32_t)code;
}

// axis 0: blocks of 32 along the columns of each row. 4 lanes per block.
__global__ void __launch_bounds__(256) quant_rows_kernel(const uint4* __restrict__ in, long long nvec, int cols,
                                                         int mma_scales, uint8_t* __restrict__ codes,
                                                         uint8_t* __restrict__ scales) {
  // nvec = rows * cols / 8; vector v covers columns [8*(v % (cols/8)), +8) of row v / (cols/8)
  const long long stride = (long long)gridDim.x * blockDim.x;
  // the loop runs while the warp's first vector is in range, so all 32 lanes stay
  // together for the shuffles; nvec is a multiple of 4, so groups are all live or all dead
  for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v - (threadIdx.x & 31) < nvec; v += stride) {
    const bool live = v < nvec;
    uint8_t sc;
    const uint2 q = mxfp8_quant8(live ? __ldg(in + v) : make_uint4(0, 0, 0, 0), &sc);
    if (live) {
      *reinterpret_cast<uint2*>(codes + v * 8) = q;
      if ((threadIdx.x & 3) == 0) {
        if (mma_scales) {
          const long long row = v / (cols >> 3);
          const int kb = (int)((v % (cols >> 3)) >> 2);
          scales[mma_scale_offset((size_t)(row >> 7), (int)(row & 127), kb, cols / 128)] = sc;
        } else {
          scales[v >> 2] = sc;
        }
      }
    }
  }
}

// Blocks of 32 rows restarting at every expert's first row, per column, for the
// weight-gradient GEMMs (contraction over the expert's rows). in/codes [R, C] (codes keep
// the layout: MN-major operands); the last block of an expert covers its remaining rows
// only (as if zero-padded). Scales go to MMA atoms numbered per expert: expert e owns
// KG_e = ceil(n_e / 128) k-groups; atom (e, column group cg, k-group kg) sits at
// (kgoff_e * C/128 + cg * KG_e + kg) * 512 with kgoff_e = sum of KG over earlier experts.
// Scale bytes of k-blocks past an expert's end (up to the next multiple of 4) are zero.
// A thread quantises 2 adjacent columns of one 32-row block (4-byte loads, 2-byte code
// stores; the block's 32 x 2 inputs stay packed in 32 registers so three blocks of 256
// threads fit per SM); blockIdx.x walks the 32-row blocks of all experts (sum of
// ceil(n_e / 32) of them), blockIdx.y the 512-column tiles of 256 threads.
__global__ void __launch_bounds__(256, 3) quant_cols_grouped_kernel(const __nv_bfloat16* __restrict__ in, int C,
                                                                 const int32_t* __restrict__ split_sizes, int E,
                                                                 uint8_t* __restrict__ codes,
                                                                 uint8_t* __restrict__ atoms) {
  extern __shared__ int32_t tabs[];   // [E+1] row offsets, [E+1] 32-row block offsets, [E+1] k-group offsets
  int32_t* roff = tabs;
  int32_t* boff = tabs + (E + 1);
  int32_t* koff = tabs + 2 * (E + 1);
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int cr = 0, cb = 0, ck = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int n = (e < E) ? split_sizes[e] : 0;
      const int nb = (n + 31) / 32, nk = (n + 127) / 128;
      int ir = n, ib = nb, ik = nk;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yr = __shfl_up_sync(0xffffffffu, ir, o);
        const int yb = __shfl_up_sync(0xffffffffu, ib, o);
        const int yk = __shfl_up_sync(0xffffffffu, ik, o);
        if (lane >= o) {
          ir += yr;
          ib += yb;
          ik += yk;
        }
      }
      if (e < E) {
        roff[e] = cr + ir - n;
        boff[e] = cb + ib - nb;
        koff[e] = ck + ik - nk;
      }
      cr += __shfl_sync(0xffffffffu, ir, 31);
      cb += __shfl_sync(0xffffffffu, ib, 31);
      ck += __shfl_sync(0xffffffffu, ik, 31);
    }
    if (lane == 0) {
      roff[E] = cr;
      boff[E] = cb;
      koff[E] = ck;
    }
  }
  __syncthreads();
  const int CG = C / 128;
  const int c0 = (blockIdx.y * blockDim.x + threadIdx.x) * 2;   // this thread's 2 columns
  if (c0 >= C) return;
  for (int blk = blockIdx.x; blk < boff[E]; blk += gridDim.x) {
    int lo = 0, hi = E - 1;   // expert owning 32-row block `blk`
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (boff[mid] <= blk) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int j = blk - boff[e];                 // block index inside the expert
    const int n = roff[e + 1] - roff[e];
    const int r0 = roff[e] + 32 * j;
    const int nrows = min(32, n - 32 * j);
    const int KG = (n + 127) / 128;
    // 32 rows x 2 columns held as packed bf16 pairs (32 registers): three blocks fit per SM
    const uint32_t* src = reinterpret_cast<const uint32_t*>(in + (size_t)r0 * C + c0);
    const size_t row_words = (size_t)C / 2;
    uint32_t raw[32];
    float amax[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      raw[i] = (i < nrows) ? __ldg(src + i * row_words) : 0u;
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[i]));
      amax[0] = fmaxf(amax[0], fabsf(f.x));
      amax[1] = fmaxf(amax[1], fabsf(f.y));
    }
    float inv[2];
    int code[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      code[q] = max((int)((__float_as_uint(amax[q]) >> 23) & 0xFF) - 8, 0);
      inv[q] = __uint_as_float((uint32_t)(254 - code[q]) << 23);
    }
    uint16_t* dst = reinterpret_cast<uint16_t*>(codes + (size_t)r0 * C + c0);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (i < nrows) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[i]));
        dst[i * row_words] =
            (uint16_t)__nv_cvt_float2_to_fp8x2(make_float2(a.x * inv[0], a.y * inv[1]), __NV_SATFINITE, __NV_E4M3);
      }
    }
    const size_t grp = (size_t)koff[e] * CG + (size_t)(c0 / 128) * KG;   // this column group's first atom
    const bool last = 32 * (j + 1) >= n;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int c = c0 + q;
      atoms[mma_scale_offset(grp, c % 128, j, 1)] = (uint8_t)code[q];
      if (last)   // the expert's last block: zero the unused bytes of its atom
        for (int jj = j + 1; jj < ((j >> 2) + 1) * 4; ++jj) atoms[mma_scale_offset(grp, c % 128, jj, 1)] = 0;
    }
  }
}

// axis 1: blocks of 32 along the rows of each column. A block of 256 threads handles a
// 32 x 256 tile of one batch matrix [rows, cols]; thread j owns column c0 + j.
// transpose_out: codes [cols, rows], scales [cols, rows/32]; else codes [rows, cols],
// scales [rows/32, cols].
__global__ void __launch_bounds__(256) quant_cols_kernel(const __nv_bfloat16* __restrict__ in, int rows, int cols,
                                                         int transpose_out, int mma_scales,
                                                         uint8_t* __restrict__ codes,
                                                         uint8_t* __restrict__ scales) {
  __shared__ __align__(16) uint8_t tile[32][256 + 16];
  __shared__ __align__(16) __nv_bfloat16 in_tile[32][256];
  const int b = blockIdx.z;
  const int r0 = blockIdx.y * 32;
  const int c0 = blockIdx.x * 256;
  const int j = threadIdx.x;
  const int c = c0 + j;
  const __nv_bfloat16* src = in + (size_t)b * rows * cols;
  uint8_t* dst = codes + (size_t)b * rows * cols;
  uint8_t* sdst = scales + (size_t)b * (rows / 32) * cols;
  float f[32];
  float amax = 0.f;
  if ((cols & 7) == 0 && (reinterpret_cast<uintptr_t>(in) & 15) == 0) {
    // the 32 x 256 input tile with 16-byte loads (a warp reads one 512-byte row segment),
    // then each thread takes its column from shared memory
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = j + 256 * i, row = idx >> 5, cv = (idx & 31) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (c0 + cv < cols) v = *reinterpret_cast<const uint4*>(src + (size_t)(r0 + row) * cols + c0 + cv);
      *reinterpret_cast<uint4*>(&in_tile[row][cv]) = v;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      f[i] = __bfloat162float(in_tile[i][j]);
      amax = fmaxf(amax, fabsf(f[i]));
    }
  } else if (c < cols) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      f[i] = __bfloat162float(src[(size_t)(r0 + i) * cols + c]);
      amax = fmaxf(amax, fabsf(f[i]));
    }
  }
  const int bexp = (int)((__float_as_uint(amax) >> 23) & 0xFF);
  const int code = max(bexp - 8, 0);
  const float inv = __uint_as_float((uint32_t)(254 - code) << 23);
  if (c < cols) {
    if (transpose_out) {
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const __nv_fp8x2_storage_t lo =
            __nv_cvt_float2_to_fp8x2(make_float2(f[4 * i] * inv, f[4 * i + 1] * inv), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
            make_float2(f[4 * i + 2] * inv, f[4 * i + 3] * inv), __NV_SATFINITE, __NV_E4M3);
        w[i] = (uint32_t)lo | ((uint32_t)hi << 16);
      }
      uint4* o = reinterpret_cast<uint4*>(dst + (size_t)c * rows + r0);
      o[0] = make_uint4(w[0], w[1], w[2], w[3]);
      o[1] = make_uint4(w[4], w[5], w[6], w[7]);
      if (mma_scales) {
        // scale atoms of the transposed matrix [cols, rows]: see mma_scale_offset
        scales[mma_scale_offset((size_t)b * (cols / 128) + c / 128, c % 128, r0 / 32, rows / 128)] = (uint8_t)code;
      } else {
        sdst[(size_t)c * (rows / 32) + (r0 / 32)] = (uint8_t)code;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const __nv_fp8x2_storage_t p =
            __nv_cvt_float2_to_fp8x2(make_float2(f[i] * inv, f[i + 1] * inv), __NV_SATFINITE, __NV_E4M3);
        tile[i][j] = (uint8_t)(p & 0xFF);
        tile[i + 1][j] = (uint8_t)(p >> 8);
      }
      sdst[(size_t)(r0 / 32) * cols + c] = (uint8_t)code;
    }
  }
  if (!transpose_out) {
    __syncthreads();
    // 32 rows x 256 bytes: each thread writes 32 bytes of one row
    const int row = threadIdx.x >> 3, part = threadIdx.x & 7;
    const int cc = c0 + part * 32;
    if (cc < cols) {
      const int n = min(32, cols - cc);
      uint8_t* o = dst + (size_t)(r0 + row) * cols + cc;
      for (int i = 0; i < n; ++i) o[i] = tile[row][part * 32 + i];
    }
  }
}

// Both MXFP8 forms of a weight tensor [batch, rows, cols] bf16 in one pass (one read):
//   T: blocks of 32 along the rows of each column, codes transposed to [batch, cols, rows]
//      with scale atoms of the transposed matrix (the K-major operand of a GEMM whose K is
//      `rows`: fc1 and fc2 forward);
//   R: blocks of 32 along the columns of each row, codes [batch, rows, cols] with atoms of
//      the [batch * rows, cols] matrix (the K-major operand of a GEMM whose K is `cols`:
//      the data-gradient GEMMs of the backward).
// The same rule as every quantiser here: E8M0 code max(biased_exp(amax) - 8, 0), elements
// times 2^(127 - code), round to nearest even, saturating. A block of 256 threads takes a
// 128 x 128 tile: 16-byte loads into shared memory, each thread quantises two 32-value
// blocks of each form into shared staging tiles, and both 128 x 128 code tiles leave as
// whole 128-byte lines (a 32-byte piece per output row scattered the stores). Row pitches
// of 272 / 144 bytes keep the column reads, the 32-value row reads and the staging stores
// free of bank conflicts. rows and cols are multiples of 128.
namespace qw {
constexpr int kInPitch = 136;    // bf16 per input row: 128 + 8
constexpr int kOutPitch = 144;   // bytes per staged code row: 128 + 16
constexpr int kSmemBytes = 128 * kInPitch * 2 + 2 * 128 * kOutPitch;
}  // namespace qw

__global__ void __launch_bounds__(256) quant_weights_both_kernel(const __nv_bfloat16* __restrict__ in, int rows,
                                                                 int cols, uint8_t* __restrict__ codes_t,
                                                                 uint8_t* __restrict__ atoms_t,
                                                                 uint8_t* __restrict__ codes_r,
                                                                 uint8_t* __restrict__ atoms_r) {
  using namespace qw;
  extern __shared__ __align__(16) uint8_t qw_smem[];
  __nv_bfloat16* tile = reinterpret_cast<__nv_bfloat16*>(qw_smem);
  uint8_t* st_t = qw_smem + 128 * kInPitch * 2;   // [128 columns][128 rows] codes of T
  uint8_t* st_r = st_t + 128 * kOutPitch;         // [128 rows][128 columns] codes of R
  const int b = blockIdx.z;
  const int r0 = blockIdx.y * 128;
  const int c0 = blockIdx.x * 128;
  const int j = threadIdx.x;
  const __nv_bfloat16* src = in + (size_t)b * rows * cols;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = j + 256 * i, row = idx >> 4, cv = (idx & 15) * 8;
    *reinterpret_cast<uint4*>(&tile[row * kInPitch + cv]) =
        *reinterpret_cast<const uint4*>(src + (size_t)(r0 + row) * cols + c0 + cv);
  }
  __syncthreads();
  float f[32];
  uint32_t w[8];
#pragma unroll 1
  for (int it = 0; it < 2; ++it) {
    // T: column c (a warp: 32 consecutive columns), rows [32 rb, +32)
    const int item = j + 256 * it, c = item & 127, rb = item >> 7;
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      f[i] = __bfloat162float(tile[(32 * rb + i) * kInPitch + c]);
      amax = fmaxf(amax, fabsf(f[i]));
    }
    const int code = max((int)((__float_as_uint(amax) >> 23) & 0xFF) - 8, 0);
    const float inv = __uint_as_float((uint32_t)(254 - code) << 23);
#pragma unroll
    for (int i = 0; i < 32; ++i) f[i] *= inv;
    pack_e4m3x16(f, *reinterpret_cast<uint32_t(*)[4]>(&w[0]));
    pack_e4m3x16(f + 16, *reinterpret_cast<uint32_t(*)[4]>(&w[4]));
    uint4* o = reinterpret_cast<uint4*>(st_t + c * kOutPitch + 32 * rb);
    o[0] = make_uint4(w[0], w[1], w[2], w[3]);
    o[1] = make_uint4(w[4], w[5], w[6], w[7]);
    const int cg = c0 + c;
    atoms_t[mma_scale_offset((size_t)b * (cols / 128) + cg / 128, cg % 128, (r0 + 32 * rb) / 32, rows / 128)] =
        (uint8_t)code;
  }
#pragma unroll 1
  for (int it = 0; it < 2; ++it) {
    // R: row r (a warp: 32 consecutive rows), columns [32 cb, +32)
    const int item = j + 256 * it, r = item & 127, cb = item >> 7;
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(&tile[r * kInPitch + 32 * cb + 8 * i]);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 p2 = __bfloat1622float2(h2[q]);
        f[8 * i + 2 * q] = p2.x;
        f[8 * i + 2 * q + 1] = p2.y;
        amax = fmaxf(amax, fmaxf(fabsf(p2.x), fabsf(p2.y)));
      }
    }
    const int code = max((int)((__float_as_uint(amax) >> 23) & 0xFF) - 8, 0);
    const float inv = __uint_as_float((uint32_t)(254 - code) << 23);
#pragma unroll
    for (int i = 0; i < 32; ++i) f[i] *= inv;
    pack_e4m3x16(f, *reinterpret_cast<uint32_t(*)[4]>(&w[0]));
    pack_e4m3x16(f + 16, *reinterpret_cast<uint32_t(*)[4]>(&w[4]));
    uint4* o = reinterpret_cast<uint4*>(st_r + r * kOutPitch + 32 * cb);
    o[0] = make_uint4(w[0], w[1], w[2], w[3]);
    o[1] = make_uint4(w[4], w[5], w[6], w[7]);
    const size_t grow = (size_t)b * rows + r0 + r;
    atoms_r[mma_scale_offset(grow >> 7, (int)(grow & 127), (c0 + 32 * cb) / 32, cols / 128)] = (uint8_t)code;
  }
  __syncthreads();
  // both 128 x 128 code tiles out as whole lines: 8 threads per 128-byte line
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = j + 256 * i, line = idx >> 3, part = (idx & 7) * 16;
    *reinterpret_cast<uint4*>(codes_t + (size_t)b * rows * cols + (size_t)(c0 + line) * rows + r0 + part) =
        *reinterpret_cast<const uint4*>(st_t + line * kOutPitch + part);
    *reinterpret_cast<uint4*>(codes_r + ((size_t)b * rows + r0 + line) * cols + c0 + part) =
        *reinterpret_cast<const uint4*>(st_r + line * kOutPitch + part);
  }
}

// Gather rows into expert order and quantise them both ways, for the two GEMMs that read
// a permuted activation or gradient in the backward (dy: fc2 dgrad along H, fc2 wgrad
// along the expert's rows; x: fc1 wgrad along the rows):
//   rows form: codes [R, C] in blocks of 32 along C, scale atoms grouped per 128-row
//     expert tile (row group sum_{e'<e} ceil(n_e'/128) + m for rows [off_e + 128 m, +128));
//   cols form: codes [R, C] in blocks of 32 rows restarting at each expert's first row,
//     scale atoms in mxfp8_quantize_grouped's layout.
// Row r of the output is src[row_token[r]]. blockIdx.x walks the 32-row blocks of all
// experts, blockIdx.y tiles of 256 columns; warp w takes 32 columns, lane l row 32 j + l
// of the expert (rows past its end count as zeros and store nothing). The atom buffers
// are zeroed by the caller (bytes of rows or blocks past an expert's end stay 0).
__global__ void __launch_bounds__(256) permute_quant_both_kernel(const __nv_bfloat16* __restrict__ src, int C,
                                                                 const int32_t* __restrict__ row_token,
                                                                 const int32_t* __restrict__ split_sizes, int E,
                                                                 uint8_t* __restrict__ rcodes,
                                                                 uint8_t* __restrict__ ratoms,
                                                                 uint8_t* __restrict__ ccodes,
                                                                 uint8_t* __restrict__ catoms) {
  extern __shared__ int32_t tabs[];   // [E+1] row offsets, [E+1] 32-row block offsets, [E+1] 128-row group offsets
  int32_t* roff = tabs;
  int32_t* boff = tabs + (E + 1);
  int32_t* koff = tabs + 2 * (E + 1);
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int cr = 0, cb = 0, ck = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int n = (e < E) ? split_sizes[e] : 0;
      const int nb = (n + 31) / 32, nk = (n + 127) / 128;
      int ir = n, ib = nb, ik = nk;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yr = __shfl_up_sync(0xffffffffu, ir, o);
        const int yb = __shfl_up_sync(0xffffffffu, ib, o);
        const int yk = __shfl_up_sync(0xffffffffu, ik, o);
        if (lane >= o) {
          ir += yr;
          ib += yb;
          ik += yk;
        }
      }
      if (e < E) {
        roff[e] = cr + ir - n;
        boff[e] = cb + ib - nb;
        koff[e] = ck + ik - nk;
      }
      cr += __shfl_sync(0xffffffffu, ir, 31);
      cb += __shfl_sync(0xffffffffu, ib, 31);
      ck += __shfl_sync(0xffffffffu, ik, 31);
    }
    if (lane == 0) {
      roff[E] = cr;
      boff[E] = cb;
      koff[E] = ck;
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = blockIdx.y * 256 + warp * 32;   // this warp's 32 columns
  if (c >= C) return;                           // warp-uniform; no block-wide sync follows
  const int CG = C / 128;
  for (int blk = blockIdx.x; blk < boff[E]; blk += gridDim.x) {
    int lo = 0, hi = E - 1;   // expert owning 32-row block `blk`
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (boff[mid] <= blk) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int j = blk - boff[e];                 // block index inside the expert
    const int n = roff[e + 1] - roff[e];
    const int rl = 32 * j + lane;                // this lane's row inside the expert
    const bool live = rl < n;
    const long long r = (long long)roff[e] + rl;
    float v[32];
    const int tok = live ? row_token[r] : -1;
    if (tok >= 0) {
      const uint4* sp = reinterpret_cast<const uint4*>(src + (size_t)tok * C + c);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 q = __ldg(sp + i);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 f2 = __bfloat1622float2(h2[t]);
          v[8 * i + 2 * t] = f2.x;
          v[8 * i + 2 * t + 1] = f2.y;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.f;
    }
    uint32_t w[8];
    if (ccodes) {
      // along the expert's rows: the warp's 32 lanes are rows 32 j .. 32 j + 31
      const int KG = (n + 127) / 128;
      const uint32_t sc = quant_cols_warp32(v, w, lane);
      catoms[mma_scale_offset((size_t)koff[e] * CG + (size_t)KG * (c / 128), (c + lane) % 128, j, 1)] =
          (uint8_t)sc;
      if (live) {
        uint4* d = reinterpret_cast<uint4*>(ccodes + r * C + c);
        d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
    if (rcodes && live) {
      // along this row's 32 columns (quant_row32 scales v in place: after the cols form)
      const uint32_t code = quant_row32(v, w);
      ratoms[mma_scale_offset((size_t)koff[e] + rl / 128, rl % 128, c / 32, CG)] = (uint8_t)code;
      uint4* d = reinterpret_cast<uint4*>(rcodes + r * C + c);
      d[0] = make_uint4(w[0], w[1], w[2], w[3]);
      d[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
  }
}

}  // namespace moe
