// Layer backward with FP8 GEMMs ("DeepSeek Technical Report: MoE
// Architecture", §3.6: activation-backward and weight-backward GEMMs in E4M3,
// activations per 1x128 tile, weights per 128x128 block, fp32 accumulation
// promoted every 128 elements; gating in BF16, weight gradients in BF16).
//
// Row space: every problem (routed expert j, then shared expert s) owns a
// segment of rows [poff[p], poff[p] + M_p) followed by zero rows up to a
// multiple of 128, so that a 128-row quantisation tile of the weight-gradient
// operands never mixes two experts.  Routed rows are the expert's tokens in
// permutation order; a shared expert's rows are all T tokens.
//
// The activation-side GEMMs (ab = X W_gu^T, dz' = dY W_down, du = dAB W_gu)
// read 1x128-quantised rows of this space; the weight-gradient GEMMs
// (dW_down = dY^T (g z), dW_gu = dAB^T X) contract over the rows, so their
// operands are quantised per 128 rows x 1 column and stored transposed
// (feature-major, K = the row space), with scales stored k-block-major.
#pragma once

#include "bwd.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "permute.cuh"

namespace moe {
namespace bwd8 {

constexpr int PAD = 128;

__host__ __device__ inline int pad128(int v) { return (v + PAD - 1) / PAD * PAD; }

struct PrepArgs {
  const int32_t* offsets;  // [N + 1] permutation offsets
  int T, d, I, Ks, N;
  int32_t* poff;           // [E + 1] segment starts (routed experts, then shared)
  int32_t* gtab;           // activation-side GEMMs: one group per problem
  int32_t* gtab_wd;        // dW_down: one group of d rows per problem
  int32_t* gtab_wgu;       // dW_gu: one group of 2I rows per problem
  int32_t* kgroup;         // [2E]: first row of the problem's segment, its 128-row blocks
  int32_t* tab_dxr;        // router GEMMs of the bf16 backward (gbwd problem tables)
  int32_t* tab_dwr;
};

__device__ inline void put_group(int32_t* gt, int n, int g, int prefix, int rows, int a_row,
                                 int expert, int c_row, int aux) {
  gt[g] = prefix;
  gt[n + 1 + g] = rows;
  gt[n + 1 + n + g] = a_row;
  gt[n + 1 + 2 * n + g] = 0;
  gt[n + 1 + 3 * n + g] = expert;
  gt[n + 1 + 4 * n + g] = c_row;
  gt[n + 1 + 5 * n + g] = aux;
}

// One block of up to 1024 threads, one thread per problem (E <= 1024).
__global__ void __launch_bounds__(1024) k_bwd8_prep(const PrepArgs a) {
  grid_dep_sync();
  __shared__ int32_t warp_tot[32];
  const int E = a.Ks + a.N;
  const int e = threadIdx.x;
  int rows = 0, padded = 0;
  if (e < E) {
    rows = e < a.N ? a.offsets[e + 1] - a.offsets[e] : a.T;
    if (rows < 0) { set_status(MOE_ERR_DEVICE_CHECK); rows = 0; }
    padded = pad128(rows);
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
    const bool routed = e < a.N;
    const int we = routed ? a.Ks + e : e - a.N;        // expert index in the weights
    const int aux = routed ? -1 : e - a.N;
    a.poff[e] = p0;
    if (e == E - 1) {
      a.poff[E] = p0 + padded;
      a.gtab[E] = (p0 + padded) / PAD;
      a.gtab_wd[E] = E * (a.d / 128);
      a.gtab_wgu[E] = E * (2 * a.I / 128);
    }
    // m-tiles of 128 rows: a segment of `padded` rows holds padded / 128 of them
    put_group(a.gtab, E, e, p0 / PAD, rows, p0, we, p0, aux);
    put_group(a.gtab_wd, E, e, e * (a.d / 128), a.d, 0, we, we * a.d, -1);
    put_group(a.gtab_wgu, E, e, e * (2 * a.I / 128), 2 * a.I, 0, we, we * 2 * a.I, -1);
    a.kgroup[2 * e] = p0;
    a.kgroup[2 * e + 1] = padded / PAD;
    if (e == 0) {
      bwd::put(a.tab_dxr, a.T, a.d, a.N, 0, 0, 0, 0, 0, 0, 0, a.T, -1);
      bwd::put(a.tab_dwr, a.N, a.d, a.T, 0, 0, 0, 0, 0, 0, 0, a.N, -1);
    }
  }
}

// One warp per token: quantise x[t] and dh[t] per 1x128 tile once and write
// the codes and scales to each of the token's rows (its K routed pairs and
// the Ks shared experts), with the row's pair, gate weight and token.
__global__ void __launch_bounds__(256) k_bwd8_gather(
    const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ dh, int T, int K,
    int Ks, int N, int d, const int32_t* __restrict__ idx, const float* __restrict__ topk_w,
    const int32_t* __restrict__ slot_of, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ poff, uint8_t* __restrict__ xq, float* __restrict__ xs,
    uint8_t* __restrict__ dhq, float* __restrict__ dhs, int32_t* __restrict__ row_pair,
    float* __restrict__ row_w, int32_t* __restrict__ row_tok) {
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
      row_tok[my_row] = t;
    } else {
      set_status(MOE_ERR_DEVICE_CHECK);
    }
  } else if (lane < K + Ks) {
    my_row = poff[N + lane - K] + t;
    row_pair[my_row] = -1;
    row_w[my_row] = 1.0f;
    row_tok[my_row] = t;
  }
  const int ng = d / 128;
  for (int g = 0; g < ng; ++g) {
    uint32_t cx, cd;
    float sx, sd;
    perm::quant_tile_1x128(x + (size_t)t * d, g, lane, cx, sx);
    perm::quant_tile_1x128(dh + (size_t)t * d, g, lane, cd, sd);
    for (int k = 0; k < K + Ks; ++k) {
      const int row = __shfl_sync(0xffffffffu, my_row, k);
      if (row < 0) continue;
      *reinterpret_cast<uint32_t*>(xq + (size_t)row * d + g * 128 + lane * 4) = cx;
      *reinterpret_cast<uint32_t*>(dhq + (size_t)row * d + g * 128 + lane * 4) = cd;
      if (lane == 0) {
        xs[(size_t)row * ng + g] = sx;
        dhs[(size_t)row * ng + g] = sd;
      }
    }
  }
}

// Block p < E marks the padding rows of problem p's segment (no token, no
// pair); block E the rows past the last segment up to the row-space bound rs.
// Grid: E + 1 blocks.
__global__ void __launch_bounds__(128) k_bwd8_pads(const int32_t* __restrict__ offsets, int N,
                                                   int T, int rs,
                                                   const int32_t* __restrict__ poff,
                                                   int32_t* __restrict__ row_pair,
                                                   float* __restrict__ row_w,
                                                   int32_t* __restrict__ row_tok) {
  grid_dep_sync();
  const int p = blockIdx.x, E = gridDim.x - 1;
  int r0 = poff[E], r1 = rs;
  if (p < E) {
    r0 = poff[p] + (p < N ? offsets[p + 1] - offsets[p] : T);
    r1 = poff[p + 1];
  }
  if (r1 > rs) r1 = rs;
  for (int r = r0 + threadIdx.x; r < r1; r += blockDim.x) {
    row_pair[r] = -1;
    row_w[r] = 0.f;
    row_tok[r] = -1;
  }
}

// Quantisation along the rows for the weight-gradient GEMMs: tiles of 128
// rows x 1 column of a bf16 [rows, C] matrix, written transposed as E4M3
// codes [C, ld] (K-major operands whose K is the row space) with the fp32
// tile scales k-block-major, scales[r / 128][C].  Scale rule as for the 1x128
// tiles: amax, amax / 448, v * (448 / amax) rounded to E4M3 (nearest even,
// saturating), all in fp32; an all-zero tile gets scale 0.
// INDIRECT: row r of the row space is row row_tok[r] of src (token order),
// zeros for row_tok[r] < 0; otherwise row r of src.
// Block: 128 rows x 64 columns, 256 threads; grid (rows / 128, C / 64).
template <bool INDIRECT>
__global__ void __launch_bounds__(256) k_quant_cols(const __nv_bfloat16* __restrict__ src,
                                                    const int32_t* __restrict__ row_tok, int C,
                                                    int ld, uint8_t* __restrict__ codes,
                                                    float* __restrict__ scales) {
  grid_dep_sync();
  __shared__ __align__(16) __nv_bfloat16 tile[128][64];
  __shared__ float part[4][64];
  const int r0 = blockIdx.x * 128, c0 = blockIdx.y * 64;
  const int tid = threadIdx.x;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int piece = tid + 256 * m, row = piece >> 3, c8 = piece & 7;
    long long srow = r0 + row;
    if (INDIRECT) srow = row_tok[r0 + row];
    uint4 v = make_uint4(0, 0, 0, 0);
    if (srow >= 0) v = *reinterpret_cast<const uint4*>(src + srow * C + c0 + c8 * 8);
    *reinterpret_cast<uint4*>(&tile[row][c8 * 8]) = v;
  }
  __syncthreads();
  const int c = tid & 63, qr = tid >> 6;        // column, quarter of the rows
  float v[32];
  float am = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    v[i] = __bfloat162float(tile[qr * 32 + i][c]);
    am = fmaxf(am, fabsf(v[i]));
  }
  part[qr][c] = am;
  __syncthreads();
  const float amax = fmaxf(fmaxf(part[0][c], part[1][c]), fmaxf(part[2][c], part[3][c]));
  const float inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 0.f;
  uint32_t w[8];
#pragma unroll
  for (int j = 0; j < 8; ++j)
    w[j] = (uint32_t)f32_to_e4m3(__fmul_rn(v[4 * j], inv)) |
           ((uint32_t)f32_to_e4m3(__fmul_rn(v[4 * j + 1], inv)) << 8) |
           ((uint32_t)f32_to_e4m3(__fmul_rn(v[4 * j + 2], inv)) << 16) |
           ((uint32_t)f32_to_e4m3(__fmul_rn(v[4 * j + 3], inv)) << 24);
  uint4* dst = reinterpret_cast<uint4*>(codes + (size_t)(c0 + c) * ld + r0 + qr * 32);
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  if (qr == 0)
    scales[(size_t)blockIdx.x * C + c0 + c] = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 0.f;
}

}  // namespace bwd8
}  // namespace moe
