// Layer backward: the padded expert-major row space, the problem tables of
// the backward GEMMs (gemm_bwd.cuh), the row gather of x and dh, and the
// gate-weight / affinity backward that turns the per-pair <dh, y> into router
// logit gradients.
//
// Follows the chain rule of the layer's output equation ("DeepSeek Technical
// Report: MoE Architecture", §1.1(2), equation [1] of §5.3) through SwiGLU
// experts, the gate weights g = c s / sum(s) (or c s) and the affinities
// (softmax over the routed experts, §2.3; sigmoid, §3.3 and equation [3] of
// §5.3).  The selection is piecewise constant, so no gradient flows through
// the chosen indices, and the selection bias (equation [4]) gets none.
//
// Padded row space: routed expert j owns rows [poff[j], poff[j] + M_j) of the
// backward's row buffers, followed by zero rows up to a multiple of 64 (the K
// block of the weight-gradient GEMMs, which contract over these rows); shared
// expert s owns rows [poff[N+s], poff[N+s] + T), padded the same way.
#pragma once

#include "common.cuh"
#include "gemm_bwd.cuh"
#include "route.cuh"

namespace moe {
namespace bwd {

constexpr int PAD = 64;

__host__ __device__ inline int pad64(int v) { return (v + PAD - 1) / PAD * PAD; }

// Problem tables of the seven backward GEMMs, one block of up to 1024 threads
// (one thread per expert; E <= 1024 is checked on the host).
//   poff [E + 1]   padded row offsets (routed experts first, then shared)
//   tabs           7 tables of E (or 1) problems, gbwd::GB_FIELDS ints each
struct PrepArgs {
  const int32_t* offsets;  // [N + 1] permutation offsets
  int T, d, I, Ks, N;
  int32_t* poff;
  int32_t* tab_ab;         // G1: ab = X W_gu^T            (E problems)
  int32_t* tab_dz;         // G2: dz' = dY W_down          (E)
  int32_t* tab_du;         // G3: du pieces = dAB W_gu     (E)
  int32_t* tab_dwd;        // G4: dW_down = dY^T ZG        (E)
  int32_t* tab_dwgu;       // G5: dW_gu = dAB^T X          (E)
  int32_t* tab_dxr;        // G6a: dx_router = dL W_r      (1)
  int32_t* tab_dwr;        // G6b: dW_r = dL^T X           (1)
};

__device__ inline void put(int32_t* t, int m, int n, int k, int amap, int am0, int ak0, int bmap,
                           int bn0, int bk0, int crow, int mpad, int aux) {
  using namespace gbwd;
  t[F_M] = m; t[F_N] = n; t[F_K] = k;
  t[F_AMAP] = amap; t[F_AM0] = am0; t[F_AK0] = ak0;
  t[F_BMAP] = bmap; t[F_BN0] = bn0; t[F_BK0] = bk0;
  t[F_CROW] = crow; t[F_MPAD] = mpad; t[F_AUX] = aux; t[F_SPARE] = 0;
}

__global__ void __launch_bounds__(1024) k_bwd_prep(const PrepArgs a) {
  grid_dep_sync();
  __shared__ int32_t warp_tot[32];
  const int E = a.Ks + a.N;
  const int e = threadIdx.x;        // 0..N-1 routed j, N..N+Ks-1 shared s
  int rows = 0, padded = 0;
  if (e < E) {
    rows = e < a.N ? a.offsets[e + 1] - a.offsets[e] : a.T;
    if (rows < 0) { set_status(MOE_ERR_DEVICE_CHECK); rows = 0; }
    padded = pad64(rows);
  }
  int incl = padded;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane_id() >= o) incl += y;
  }
  if (lane_id() == 31) warp_tot[warp_id()] = incl;
  __syncthreads();
  if (warp_id() == 0) {
    const int nw = blockDim.x / 32;
    const int wv = lane_id() < nw ? warp_tot[lane_id()] : 0;
    int wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane_id() >= o) wi += y;
    }
    if (lane_id() < nw) warp_tot[lane_id()] = wi - wv;
  }
  __syncthreads();
  const int p0 = incl - padded + warp_tot[warp_id()];
  if (e < E) {
    a.poff[e] = p0;
    if (e == E - 1) a.poff[E] = p0 + padded;
    const int d = a.d, I = a.I, T = a.T;
    const bool routed = e < a.N;
    const int we = routed ? a.Ks + e : e - a.N;          // expert index in w_gu / w_down
    const int aux = routed ? -1 : e - a.N;
    const int F = gbwd::GB_FIELDS;
    // A / B maps: 0 = the token-order tensor (x or dh), 1 = the padded row buffer
    const int am = routed ? 1 : 0, am0 = routed ? p0 : 0;
    put(a.tab_ab + e * F, rows, 2 * I, d, am, am0, 0, 0, we * 2 * I, 0, p0, padded, aux);
    put(a.tab_dz + e * F, rows, I, d, am, am0, 0, 0, 0, we * d, p0, padded, aux);
    // the problem's first row among the forward's H rows (routed expert j:
    // offsets[j]; shared expert s: R + s T), where saved pre-activations live
    a.tab_dz[e * F + gbwd::F_SPARE] = routed ? a.offsets[e] : a.offsets[a.N] + (e - a.N) * T;
    put(a.tab_du + e * F, rows, d, 2 * I, 0, p0, 0, 0, 0, we * 2 * I, p0, padded, aux);
    // weight gradients contract over the expert's rows (zero rows pad them to 64)
    put(a.tab_dwd + e * F, d, I, routed ? padded : T, am, 0, routed ? p0 : 0, 0, 0, p0, we * d,
        d, aux);
    put(a.tab_dwgu + e * F, 2 * I, d, routed ? padded : T, 0, 0, p0, am, 0, routed ? p0 : 0,
        we * 2 * I, 2 * I, aux);
    if (e == 0) {
      put(a.tab_dxr, T, d, a.N, 0, 0, 0, 0, 0, 0, 0, T, -1);
      put(a.tab_dwr, a.N, d, T, 0, 0, 0, 0, 0, 0, 0, a.N, -1);
    }
  }
}

// Token-centric gather into the padded row space: each warp reads x[t] and
// dh[t] once and writes them to the padded rows of the token's K pairs, with
// the pair index and its gate weight.
__global__ void __launch_bounds__(256) k_bwd_gather(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ dh, int T, int K, int d,
    const int32_t* __restrict__ idx, const float* __restrict__ topk_w,
    const int32_t* __restrict__ slot_of, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ poff, int N, __nv_bfloat16* __restrict__ x_pad,
    __nv_bfloat16* __restrict__ dh_pad, int32_t* __restrict__ row_pair,
    float* __restrict__ row_w) {
  grid_dep_sync();
  const int t = blockIdx.x * 8 + warp_id();
  if (t >= T) return;
  const int lane = lane_id();
  int my_row = -1;
  if (lane < K) {
    const int e = idx[(size_t)t * K + lane];
    const int slot = slot_of[(size_t)t * K + lane];
    if ((unsigned)e < (unsigned)N && slot >= offsets[e] && slot < offsets[e + 1]) {
      my_row = poff[e] + (slot - offsets[e]);
      row_pair[my_row] = t * K + lane;
      row_w[my_row] = topk_w[(size_t)t * K + lane];
    } else {
      set_status(MOE_ERR_DEVICE_CHECK);
    }
  }
  const uint4* sx = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  const uint4* sd = reinterpret_cast<const uint4*>(dh + (size_t)t * d);
  const int nvec = d / 8;
  for (int c0 = 0; c0 < nvec; c0 += 32) {
    const int c = c0 + lane;
    const bool in = c < nvec;
    uint4 vx = make_uint4(0, 0, 0, 0), vd = vx;
    if (in) { vx = __ldg(sx + c); vd = __ldg(sd + c); }
    for (int k = 0; k < K; ++k) {
      const int row = __shfl_sync(0xffffffffu, my_row, k);
      if (!in || row < 0) continue;
      reinterpret_cast<uint4*>(x_pad + (size_t)row * d)[c] = vx;
      reinterpret_cast<uint4*>(dh_pad + (size_t)row * d)[c] = vd;
    }
  }
}

// Zero the padding rows of the routed experts' segments (x_pad, dh_pad) and
// mark them in row_pair / row_w.  Block j handles routed expert j.
__global__ void __launch_bounds__(256) k_bwd_zero_pads(const int32_t* __restrict__ offsets,
                                                       const int32_t* __restrict__ poff, int d,
                                                       __nv_bfloat16* __restrict__ x_pad,
                                                       __nv_bfloat16* __restrict__ dh_pad,
                                                       int32_t* __restrict__ row_pair,
                                                       float* __restrict__ row_w) {
  grid_dep_sync();
  const int j = blockIdx.x;
  const int rows = offsets[j + 1] - offsets[j];
  const int r0 = poff[j] + rows, r1 = poff[j + 1];
  const int nvec = d / 8;
  for (int i = threadIdx.x; i < (r1 - r0) * nvec; i += blockDim.x) {
    const int r = r0 + i / nvec, c = i % nvec;
    reinterpret_cast<uint4*>(x_pad + (size_t)r * d)[c] = make_uint4(0, 0, 0, 0);
    reinterpret_cast<uint4*>(dh_pad + (size_t)r * d)[c] = make_uint4(0, 0, 0, 0);
  }
  for (int r = r0 + threadIdx.x; r < r1; r += blockDim.x) {
    row_pair[r] = -1;
    row_w[r] = 0.f;
  }
}

// Gate-weight and affinity backward, one warp per token.
//   dg_k  = <dh_t, y_{t,k}> = sum over the feature tiles of the partials the
//           dz' GEMM left for the pair's padded row (fixed order)
//   ds_k  = c (dg_k - sum_k' dg_k' s_k' / S) / S   (renorm, S = sum_k s_k)
//         = c dg_k                                  (no renorm)
//   dl    = ds s (1 - s)                            (sigmoid)
//         = s (ds - <ds, s>)                        (softmax over the N experts)
// with s recomputed from the router logits exactly as the forward computes it.
// dl is written as bf16 [T, N] (the A operand of the router-gradient GEMMs).
template <int VPL>
__global__ void __launch_bounds__(256) k_gate_bwd(
    const float* __restrict__ logits, const route::Params p, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ slot_of, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ poff, const float* __restrict__ dgp, int n_it,
    __nv_bfloat16* __restrict__ dl) {
  grid_dep_sync();
  const int t = blockIdx.x * 8 + warp_id();
  if (t >= p.T) return;
  const int lane = lane_id();
  float l[VPL], s[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int e = lane * VPL + j;
    l[j] = e < p.N ? logits[(size_t)t * p.N + e] : -INFINITY;
  }
  route::affinity_lane<VPL>(l, p, s);
  // the K selected experts: lane k < K holds pick k's s and dg
  int my_e = -1;
  float my_dg = 0.f;
  if (lane < p.K) {
    my_e = idx[(size_t)t * p.K + lane];
    if ((unsigned)my_e < (unsigned)p.N) {
      const int slot = slot_of[(size_t)t * p.K + lane];
      const int row = poff[my_e] + (slot - offsets[my_e]);
      for (int i = 0; i < n_it; ++i) my_dg += dgp[(size_t)row * n_it + i];
    } else {
      my_e = -1;
    }
  }
  float my_s = 0.f;
  for (int k = 0; k < p.K; ++k) {
    const int e = __shfl_sync(0xffffffffu, my_e, k);
    float v = 0.f;
#pragma unroll
    for (int j = 0; j < VPL; ++j)
      if (lane * VPL + j == e) v = s[j];
    // the lane holding expert e broadcasts its s
    const float sv = __shfl_sync(0xffffffffu, v, e >= 0 ? e / VPL : 0);
    if (lane == k) my_s = e >= 0 ? sv : 0.f;
  }
  // gate-weight backward
  float ssum = 0.f, dgs = 0.f;
  for (int k = 0; k < p.K; ++k) {
    const float sk = __shfl_sync(0xffffffffu, my_s, k);
    const float gk = __shfl_sync(0xffffffffu, my_dg, k);
    ssum += sk;
    dgs = fmaf(gk, sk, dgs);
  }
  float my_ds;
  if (p.renorm) my_ds = p.scale * (my_dg - dgs / ssum) / ssum;
  else my_ds = p.scale * my_dg;
  // dense ds over this lane's experts
  float ds[VPL];
#pragma unroll
  for (int j = 0; j < VPL; ++j) ds[j] = 0.f;
  float dot = 0.f;   // <ds, s>
  for (int k = 0; k < p.K; ++k) {
    const int e = __shfl_sync(0xffffffffu, my_e, k);
    const float dk = __shfl_sync(0xffffffffu, my_ds, k);
    const float sk = __shfl_sync(0xffffffffu, my_s, k);
    dot = fmaf(dk, sk, dot);
#pragma unroll
    for (int j = 0; j < VPL; ++j)
      if (lane * VPL + j == e) ds[j] += dk;
  }
#pragma unroll
  for (int j = 0; j < VPL; ++j) {
    const int e = lane * VPL + j;
    if (e >= p.N) continue;
    float g;
    if (p.gate == MOE_GATE_SOFTMAX) g = s[j] * (ds[j] - dot);
    else g = ds[j] * s[j] * (1.0f - s[j]);
    dl[(size_t)t * p.N + e] = __float2bfloat16_rn(g);
  }
}

}  // namespace bwd
}  // namespace moe
