// Gating: affinities, bias-for-selection keys, group limit, top-K and gate
// weights, one warp per token with shuffle reductions.  The expert counts are
// not taken here: they are the totals of the permutation's per-chunk
// histogram (k_hist / k_scan), which costs no global atomics.
//
// Follows "DeepSeek Technical Report: MoE Architecture": §2.3 (softmax gate
// over the routed experts, then TopK), §3.3 and equations [3]/[4] of §5.3
// (sigmoid affinity; the bias b_i enters only the selection key s_i + b_i and
// the gate value is the unbiased s_i).  Group limit: experts form n_group
// contiguous groups scored by the sum of their two largest keys, and only the
// topk_group best groups stay eligible.  Ties go to the lower index.
#pragma once

#include "common.cuh"

namespace moe {
namespace route {

constexpr int MAXK = 16;   // largest top-K accepted

struct Params {
  int T, N, K, gate, renorm, n_group, topk_group;
  float scale;
};

// Unsigned image of a float that orders like the float (-0 folded into +0),
// so a warp arg-max is one redux.sync max plus a ballot for the lowest lane.
__device__ __forceinline__ uint32_t ord_key(float v) {
  const uint32_t u = __float_as_uint(v + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Affinities of one token in fp32: lane l holds experts l*VPL .. +VPL-1.
// softmax over the N routed experts (max-subtracted, butterfly sums) or the
// element-wise sigmoid; entries with index >= N get 0.
template <int VPL>
__device__ __forceinline__ void affinity_lane(const float (&l)[VPL], const Params& p,
                                              float (&s)[VPL]) {
  const int lane = lane_id();
  if (p.gate == MOE_GATE_SOFTMAX) {
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < VPL; ++j)
      if (lane * VPL + j < p.N) m = fmaxf(m, l[j]);
    m = warp_max(m);
    float z = 0.f;
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      s[j] = (lane * VPL + j < p.N) ? expf(l[j] - m) : 0.f;
      z += s[j];
    }
    z = warp_sum(z);
#pragma unroll
    for (int j = 0; j < VPL; ++j) s[j] = s[j] / z;
  } else {
#pragma unroll
    for (int j = 0; j < VPL; ++j)
      s[j] = (lane * VPL + j < p.N) ? 1.0f / (1.0f + expf(-l[j])) : 0.f;
  }
}

// Put the better of list positions a < b first: the larger key image, and
// among equal keys the lower expert (j ascending within a lane).
template <int VPL>
__device__ __forceinline__ void cas_pick(uint32_t (&ok)[VPL], int (&jj)[VPL], float (&ss)[VPL],
                                         int a, int b) {
  const bool sw = ok[b] > ok[a] || (ok[b] == ok[a] && jj[b] < jj[a]);
  const uint32_t o0 = ok[a], o1 = ok[b];
  const int j0 = jj[a], j1 = jj[b];
  const float s0 = ss[a], s1 = ss[b];
  ok[a] = sw ? o1 : o0; ok[b] = sw ? o0 : o1;
  jj[a] = sw ? j1 : j0; jj[b] = sw ? j0 : j1;
  ss[a] = sw ? s1 : s0; ss[b] = sw ? s0 : s1;
}

// Route one token given its N logits spread over the warp: lane l holds the
// logits of experts l*VPL .. l*VPL+VPL-1 (entries with index >= N are ignored).
//   1. affinities s (softmax or sigmoid) and selection keys s + b;
//   2. group limit: each group's score is the sum of its two largest keys;
//      a group is kept when fewer than topk_group groups rank above it
//      (larger score, or equal score and lower index), and the experts of the
//      other groups drop out;
//   3. each lane sorts its eligible experts by (key desc, index asc) into a
//      list; the K picks then each take the largest list head over the warp
//      (one redux.sync max on the keys' order-preserving images) and, among
//      equal keys, the lowest lane -- experts are lane-major, so that is the
//      lowest index -- and that lane drops its head;
//   4. weights in pick order: g_k = scale * s_k (/ sum of the picked s when
//      renorm); lane k writes pick k.
template <int VPL>
__device__ __forceinline__ void route_token(const float (&l)[VPL], const float* __restrict__ bias,
                                            const Params& p, int t, int32_t* __restrict__ topk_idx,
                                            float* __restrict__ topk_w) {
  const int lane = lane_id();
  float s[VPL], key[VPL];
  affinity_lane<VPL>(l, p, s);
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int e = lane * VPL + j;
    key[j] = (e < p.N) ? (bias ? s[j] + bias[e] : s[j]) : -INFINITY;
  }
  uint32_t ok[VPL];   // order-preserving key images; 0 = not eligible
#pragma unroll
  for (int j = 0; j < VPL; ++j) ok[j] = (lane * VPL + j < p.N) ? ord_key(key[j]) : 0u;

  if (p.n_group > 1) {
    const int gsz = p.N / p.n_group;
    // lane g (< n_group) ends up holding the score of group g
    float my_gscore = -INFINITY;
    const int lpg = gsz / VPL;  // lanes per group when groups are whole lanes
    if (gsz % VPL == 0 && lpg <= 32 && (lpg & (lpg - 1)) == 0) {
      // every lane's VPL experts lie in one group: per-lane top-2, then a
      // butterfly merge over the group's lpg lanes
      float b1 = -INFINITY, b2 = -INFINITY;
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        const float v = key[j];
        if (v > b1) { b2 = b1; b1 = v; } else if (v > b2) { b2 = v; }
      }
      for (int o = 1; o < lpg; o <<= 1) {
        const float o1 = __shfl_xor_sync(0xffffffffu, b1, o);
        const float o2 = __shfl_xor_sync(0xffffffffu, b2, o);
        const float hi = fmaxf(b1, o1);
        const float lo = fmaxf(fminf(b1, o1), fmaxf(b2, o2));
        b1 = hi;
        b2 = lo;
      }
      const float gs = b1 + b2;  // the group score, held by each of its lanes
      // move group g's score to lane g
      const int src = lane * lpg;
      const float moved = __shfl_sync(0xffffffffu, gs, src < 32 ? src : 0);
      if (lane < p.n_group) my_gscore = moved;
    } else {
      for (int g = 0; g < p.n_group; ++g) {
        float b1 = -INFINITY, b2 = -INFINITY;   // two largest keys of this lane in group g
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
          const int e = lane * VPL + j;
          if (e < p.N && e / gsz == g) {
            const float v = key[j];
            if (v > b1) { b2 = b1; b1 = v; } else if (v > b2) { b2 = v; }
          }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          const float o1 = __shfl_xor_sync(0xffffffffu, b1, o);
          const float o2 = __shfl_xor_sync(0xffffffffu, b2, o);
          const float hi = fmaxf(b1, o1);
          const float lo = fmaxf(fminf(b1, o1), fmaxf(b2, o2));
          b1 = hi;
          b2 = lo;
        }
        if (lane == g) my_gscore = b1 + b2;
      }
    }
    // rank of each group: groups with a larger score, or an equal score and a
    // lower index, come first; the topk_group first groups are kept
    int rank = 0;
    for (int g = 0; g < p.n_group; ++g) {
      const float o = __shfl_sync(0xffffffffu, my_gscore, g);
      rank += (o > my_gscore || (o == my_gscore && g < lane)) ? 1 : 0;
    }
    const uint32_t keep = __ballot_sync(0xffffffffu, lane < p.n_group && rank < p.topk_group);
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int e = lane * VPL + j;
      if (e < p.N && !((keep >> (e / gsz)) & 1u)) ok[j] = 0u;
    }
  }

  // per-lane list, sorted by (key desc, index asc): odd-even transposition
  int jj[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) jj[j] = j;
#pragma unroll
  for (int r = 0; r < VPL; ++r)
#pragma unroll
    for (int i = r & 1; i + 1 < VPL; i += 2) cas_pick<VPL>(ok, jj, s, i, i + 1);

  int my_i = 0;
  float my_s = 0.f, denom = 0.f;
#pragma unroll 1
  for (int k = 0; k < p.K; ++k) {
    const uint32_t mx = __reduce_max_sync(0xffffffffu, ok[0]);
    const uint32_t who = __ballot_sync(0xffffffffu, ok[0] == mx);
    const int wl = __ffs(who) - 1;
    const int bi = __shfl_sync(0xffffffffu, lane * VPL + jj[0], wl);
    const float sv = __shfl_sync(0xffffffffu, s[0], wl);
    if (lane == wl) {
#pragma unroll
      for (int j = 0; j + 1 < VPL; ++j) { ok[j] = ok[j + 1]; jj[j] = jj[j + 1]; s[j] = s[j + 1]; }
      ok[VPL - 1] = 0u;
    }
    if (lane == k) { my_i = bi; my_s = sv; }
    denom += sv;
  }
  if (!p.renorm) denom = 1.0f;
  if (lane < p.K) {
    const float g = p.renorm ? my_s / denom * p.scale : my_s * p.scale;
    topk_idx[(size_t)t * p.K + lane] = my_i;
    topk_w[(size_t)t * p.K + lane] = g;
  }
}

// Top-K over precomputed fp32 logits [T, N] (row stride N).
template <int VPL>
__global__ void __launch_bounds__(256) k_topk(const float* __restrict__ logits,
                                              const float* __restrict__ bias, const Params p,
                                              int32_t* __restrict__ topk_idx,
                                              float* __restrict__ topk_w) {
  grid_dep_sync();
  const int t = blockIdx.x * 8 + warp_id();
  if (t >= p.T) return;
  const float* row = logits + (size_t)t * p.N;
  float l[VPL];
  const int e0 = lane_id() * VPL;
  if (VPL % 4 == 0 && (p.N & 3) == 0 && e0 + VPL <= p.N) {
    // rows start 16-byte aligned when N is a multiple of 4
#pragma unroll
    for (int j = 0; j < VPL; j += 4) {
      const float4 q = *reinterpret_cast<const float4*>(row + e0 + j);
      l[j] = q.x; l[j + 1] = q.y; l[j + 2] = q.z; l[j + 3] = q.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < VPL; ++j) l[j] = e0 + j < p.N ? row[e0 + j] : -INFINITY;
  }
  route_token<VPL>(l, bias, p, t, topk_idx, topk_w);
}

// fp32 gating: router logits on CUDA cores in fp32 (one warp per token, a
// butterfly warp sum per expert), then the same selection.
template <int VPL>
__global__ void __launch_bounds__(256) k_route_f32(const float* __restrict__ x,
                                                   const float* __restrict__ w_r, int d,
                                                   const float* __restrict__ bias, const Params p,
                                                   int32_t* __restrict__ topk_idx,
                                                   float* __restrict__ topk_w) {
  grid_dep_sync();
  const int t = blockIdx.x * 8 + warp_id();
  if (t >= p.T) return;
  const int lane = lane_id();
  const float* xr = x + (size_t)t * d;
  float l[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) l[j] = -INFINITY;
  for (int e = 0; e < p.N; ++e) {
    const float* wr = w_r + (size_t)e * d;
    float acc = 0.f;
    for (int c = lane; c < d; c += 32) acc = fmaf(xr[c], wr[c], acc);
    acc = warp_sum(acc);
#pragma unroll
    for (int j = 0; j < VPL; ++j)
      if (lane * VPL + j == e) l[j] = acc;
  }
  route_token<VPL>(l, bias, p, t, topk_idx, topk_w);
}

// Affinities of every token for every routed expert (for balance statistics):
// s_out [T, N] fp32 from precomputed logits [T, N].
template <int VPL>
__global__ void __launch_bounds__(256) k_affinity(const float* __restrict__ logits, const Params p,
                                                  float* __restrict__ s_out) {
  const int t = blockIdx.x * 8 + warp_id();
  if (t >= p.T) return;
  float l[VPL], s[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int e = lane_id() * VPL + j;
    l[j] = e < p.N ? logits[(size_t)t * p.N + e] : -INFINITY;
  }
  affinity_lane<VPL>(l, p, s);
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int e = lane_id() * VPL + j;
    if (e < p.N) s_out[(size_t)t * p.N + e] = s[j];
  }
}

// The same for the fp32 layer, with the logits computed in fp32 on CUDA cores.
template <int VPL>
__global__ void __launch_bounds__(256) k_affinity_f32(const float* __restrict__ x,
                                                      const float* __restrict__ w_r, int d,
                                                      const Params p, float* __restrict__ s_out) {
  const int t = blockIdx.x * 8 + warp_id();
  if (t >= p.T) return;
  const int lane = lane_id();
  const float* xr = x + (size_t)t * d;
  float l[VPL], s[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) l[j] = -INFINITY;
  for (int e = 0; e < p.N; ++e) {
    const float* wr = w_r + (size_t)e * d;
    float acc = 0.f;
    for (int c = lane; c < d; c += 32) acc = fmaf(xr[c], wr[c], acc);
    acc = warp_sum(acc);
#pragma unroll
    for (int j = 0; j < VPL; ++j)
      if (lane * VPL + j == e) l[j] = acc;
  }
  affinity_lane<VPL>(l, p, s);
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int e = lane * VPL + j;
    if (e < p.N) s_out[(size_t)t * p.N + e] = s[j];
  }
}

// Per sequence q of L consecutive tokens and routed expert i:
//   f[q, i] = (tokens of q that selected i) / L,  P[q, i] = (sum of s[t, i] over q) / L.
// Block (q, 32-expert slice): lane = expert, the 8 warps split the sequence's
// tokens into contiguous ranges; the partial sums are combined in warp order,
// so the result is the same on every run.
__global__ void __launch_bounds__(256) k_balance_stats(const float* __restrict__ s,
                                                       const int32_t* __restrict__ idx, int T,
                                                       int N, int K, int L,
                                                       float* __restrict__ f_out,
                                                       float* __restrict__ p_out) {
  __shared__ float psum[8][32];
  __shared__ int cnt[32];
  const int q = blockIdx.x, e0 = blockIdx.y * 32;
  const int lane = lane_id(), w = warp_id();
  if (threadIdx.x < 32) cnt[threadIdx.x] = 0;
  __syncthreads();
  const int per = (L + 7) / 8;
  const int ta = q * L + w * per, tb = min(q * L + L, ta + per);
  const int e = e0 + lane;
  float acc = 0.f;
  for (int t = ta; t < tb; ++t) {
    if (e < N) acc += s[(size_t)t * N + e];
    if (lane < K) {
      const int j = idx[(size_t)t * K + lane] - e0;
      if ((unsigned)j < 32u) atomicAdd(&cnt[j], 1);
    }
  }
  psum[w][lane] = acc;
  __syncthreads();
  if (w == 0 && e < N) {
    float tot = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) tot += psum[j][lane];
    p_out[(size_t)q * N + e] = tot / (float)L;
    f_out[(size_t)q * N + e] = (float)cnt[lane] / (float)L;
  }
}

// One step of the auxiliary-loss-free rule: b_i -= gamma above the mean load
// T*K/N, += gamma below it (compared exactly in integers), in fp32.
__global__ void k_bias_update(const int32_t* __restrict__ counts, float* __restrict__ bias, int N,
                              long long total, float gamma) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < N; i += gridDim.x * blockDim.x) {
    const long long c = (long long)counts[i] * N;
    if (c > total) bias[i] = __fsub_rn(bias[i], gamma);
    else if (c < total) bias[i] = __fadd_rn(bias[i], gamma);
  }
}

__global__ void k_zero_i32(int32_t* p, int n) {
  grid_dep_sync();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p[i] = 0;
}

}  // namespace route
}  // namespace moe
