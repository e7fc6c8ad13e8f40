// Gating: affinities, bias-for-selection keys, group limit, top-K and gate
// weights, one warp per token with shuffle reductions.
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

constexpr int MAXK = 16;

struct Params {
  int T, N, K, gate, renorm, n_group, topk_group;
  float scale;
};

// (key desc, index asc) ordering of candidates
__device__ __forceinline__ bool better(float v, int i, float ov, int oi) {
  return ov > v || (ov == v && oi < i);
}

// Warp arg-max over (key, index) carrying the affinity along.
__device__ __forceinline__ void warp_argmax(float& v, int& i, float& s) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    const float os = __shfl_xor_sync(0xffffffffu, s, o);
    if (better(v, i, ov, oi)) { v = ov; i = oi; s = os; }
  }
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

// Route one token given its N logits spread over the warp: lane l holds the
// logits of experts l*VPL .. l*VPL+VPL-1 (entries with index >= N are ignored).
template <int VPL>
__device__ __forceinline__ void route_token(const float (&l)[VPL], const float* __restrict__ bias,
                                            const Params& p, int t, int32_t* __restrict__ topk_idx,
                                            float* __restrict__ topk_w,
                                            int32_t* __restrict__ counts) {
  const int lane = lane_id();
  float s[VPL], key[VPL];
  affinity_lane<VPL>(l, p, s);
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int e = lane * VPL + j;
    key[j] = (e < p.N) ? (bias ? s[j] + bias[e] : s[j]) : -INFINITY;
  }

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
    // keep the topk_group best groups (score desc, group asc)
    uint32_t keep = 0;
    for (int r = 0; r < p.topk_group; ++r) {
      const bool cand = lane < p.n_group && !((keep >> lane) & 1u);
      float v = cand ? my_gscore : -INFINITY;
      int gi = cand ? lane : (1 << 20);
      float unused = 0.f;
      warp_argmax(v, gi, unused);
      if (gi < 32) keep |= 1u << gi;
    }
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
      const int e = lane * VPL + j;
      if (e < p.N && !((keep >> (e / gsz)) & 1u)) key[j] = -INFINITY;
    }
  }

  // top-K by (key desc, index asc)
  int sel_i[MAXK];
  float sel_s[MAXK];
  uint32_t taken = 0;
#pragma unroll
  for (int k = 0; k < MAXK; ++k) {
    sel_i[k] = 0;
    sel_s[k] = 0.f;
    if (k < p.K) {
      float v = -INFINITY, sv = 0.f;
      int bi = 1 << 20;
#pragma unroll
      for (int j = 0; j < VPL; ++j) {
        const int e = lane * VPL + j;
        if (e < p.N && !((taken >> j) & 1u) && better(v, bi, key[j], e)) {
          v = key[j];
          bi = e;
          sv = s[j];
        }
      }
      warp_argmax(v, bi, sv);
      sel_i[k] = bi;
      sel_s[k] = sv;
      if (bi / VPL == lane) taken |= 1u << (bi - lane * VPL);
    }
  }
  float denom = 1.0f;
  if (p.renorm) {
    denom = 0.f;
#pragma unroll
    for (int k = 0; k < MAXK; ++k)
      if (k < p.K) denom += sel_s[k];
  }
  int my_i = 0;
  float my_s = 0.f;
#pragma unroll
  for (int k = 0; k < MAXK; ++k)
    if (lane == k) { my_i = sel_i[k]; my_s = sel_s[k]; }
  if (lane < p.K) {
    const float g = p.renorm ? my_s / denom * p.scale : my_s * p.scale;
    topk_idx[(size_t)t * p.K + lane] = my_i;
    topk_w[(size_t)t * p.K + lane] = g;
    atomicAdd(&counts[my_i], 1);
  }
}

// Top-K over precomputed fp32 logits [T, N] (row stride N).
template <int VPL>
__global__ void __launch_bounds__(256) k_topk(const float* __restrict__ logits,
                                              const float* __restrict__ bias, const Params p,
                                              int32_t* __restrict__ topk_idx,
                                              float* __restrict__ topk_w,
                                              int32_t* __restrict__ counts) {
  const int t = blockIdx.x * 8 + warp_id();
  if (t >= p.T) return;
  const float* row = logits + (size_t)t * p.N;
  float l[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int e = lane_id() * VPL + j;
    l[j] = e < p.N ? row[e] : -INFINITY;
  }
  route_token<VPL>(l, bias, p, t, topk_idx, topk_w, counts);
}

// fp32 gating: router logits on CUDA cores in fp32 (one warp per token, a
// butterfly warp sum per expert), then the same selection.
template <int VPL>
__global__ void __launch_bounds__(256) k_route_f32(const float* __restrict__ x,
                                                   const float* __restrict__ w_r, int d,
                                                   const float* __restrict__ bias, const Params p,
                                                   int32_t* __restrict__ topk_idx,
                                                   float* __restrict__ topk_w,
                                                   int32_t* __restrict__ counts) {
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
  route_token<VPL>(l, bias, p, t, topk_idx, topk_w, counts);
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
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p[i] = 0;
}

}  // namespace route
}  // namespace moe
