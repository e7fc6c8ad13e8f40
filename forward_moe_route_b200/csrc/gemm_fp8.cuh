// Grouped GEMM with FP8 E4M3 operands and fine-grained fp32 scales.
//
// Follows "DeepSeek Technical Report: MoE Architecture", §3.6 (FP8 mixed
// precision): E4M3 operands, activations scaled per 1x128 tile, weights per
// 128x128 block, fp32 accumulation with promotion every 128 elements of K.
//
// Each 128-element block of K (one 128-byte k-block) is multiplied on the
// tensor cores into a fresh TMEM partial P_kb (tcgen05.mma kind::f8f6f4, fp32
// accumulation).  The epilogue warps promote it on the CUDA cores:
//   acc += (sa[row, kb] * sb[col block, kb]) * P_kb
// so every k-block carries its own activation and weight scale.  Two TMEM
// partials (2 x 256 columns) let the MMA of k-block kb+1 overlap the promotion
// of kb.
//
// Warp roles (640 threads, one CTA per SM):
//   warp 0      TMA producer (and TMEM allocator)
//   warp 1      MMA issuer
//   warps 2, 3  idle
//   warps 4..19 16 promotion/epilogue warps: warp w owns TMEM lane quadrant
//               w % 4 (32 rows) and the 64-column slice (w - 4) / 4 of the tile.
// Registers: the register file is split evenly over the SM's four
// sub-partitions and warp w lives on sub-partition w % 4, so with 20 warps
// each sub-partition holds 5 and the launch gets 96 registers a thread.  The
// first warpgroup then drops to 32 (setmaxnreg.dec) and the four epilogue
// warpgroups rise to 112 (setmaxnreg.inc): 128 x 32 + 512 x 112 = 640 x 96.
// The extra registers hold two TMEM loads in flight per warp during the
// promotion (64 accumulators + 32 staging), which halves the number of
// TMEM round trips per k-block.
// Tile: 128 rows x 256 accumulator columns.
//   GEMM1 (SWIGLU): the B tile holds W_gate and W_up rows interleaved in
//     chunks of 32 (gate 0-31, up 0-31, gate 32-63, up 32-63, ...), so each
//     64-column slice holds matching gate and up columns; the epilogue forms
//     H = SiLU(gate) * up for 128 H columns (one 1x128 quantisation tile per
//     row), exchanges the per-slice amax through shared memory, and writes E4M3
//     codes plus the fp32 tile scale.
//   GEMM2 (SCATTER): 256 output columns, times the gate weight, bf16 rows
//     scattered to the token-major slots (weight 1 without topk_w: the
//     backward's du pieces).
//   Backward (same pipeline): BF16_OUT stores the tile as bf16 rows (the
//     recomputed a | b); SWIGLU_BWD turns dz' = dY W_down into g z, [da | db]
//     and per-64-feature partials of <dz', z>.
//   Weight-gradient mode (template WG, dW = sum over an expert's rows): each
//     group contracts over its own K range, both operands carry a scale per
//     row and k-block, so the promotion multiplies every accumulator column
//     by its own scale; tiles are 128 x 128 (32 columns a warp) and each warp
//     writes its rows through a shared-memory staging buffer.
#pragma once

#include "common.cuh"
#include "gemm.cuh"

namespace moe {
namespace gemm8 {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int KB = 128;              // bytes = elements of K per k-block
constexpr int NUM_THREADS = 640;
constexpr int EPI_WARP0 = 4;
constexpr int LAUNCH_REGS = 96;      // registers a thread at launch (host checks)
constexpr int CTRL_REGS = 32;        // first warpgroup after setmaxnreg.dec
constexpr int EPI_REGS = 112;        // epilogue warpgroups after setmaxnreg.inc
static_assert(128 * CTRL_REGS + (NUM_THREADS - 128) * EPI_REGS == NUM_THREADS * LAUNCH_REGS,
              "register split must add up to the launch allocation");
constexpr int NUM_EPI = NUM_THREADS - EPI_WARP0 * 32;   // 512
constexpr int TMEM_COLS = 512;       // two 256-column partials

enum Epi { EPI_F32_STORE = 0, EPI_SWIGLU_Q = 1, EPI_SCATTER = 2, EPI_BF16_OUT = 3,
           EPI_SWIGLU_BWD = 4 };

struct Args {
  gemm::GroupTab gt;
  int n_tiles_n;
  int num_kb;
  int kb_elems;              // elements of K per k-block (128 E4M3, 64 bf16)
  int b_rows_per_expert;     // rows of B per expert (2I for GEMM1, d for GEMM2)
  int b_up_off;              // GEMM1: row offset of W_up inside an expert (I)
  int a_from_crow;           // GEMM2 reads A (H) rows from c_row
  int stages;
  uint32_t idesc;
  // scales
  const float* a_scale;      // [A rows, num_kb]
  int a_rows;                // rows of the A tensor (scales beyond it read as 0)
  const float* b_scale;      // [E, b_rows_per_expert/128, num_kb]
  // GEMM1 outputs
  uint8_t* hq;               // [H rows, I] E4M3
  float* hs;                 // [H rows, I/128]
  int inter;                 // I
  // GEMM2 outputs
  __nv_bfloat16* y;          // [T*(K+Ks), d]
  int d;
  const int* pair_of;
  const float* topk_w;
  int K, Ks;
  // F32_STORE (router logits): out [rows, out_ld] fp32, columns < out_cols
  float* out;
  int out_ld, out_cols;
  int* zero_ptr;             // prologue: zero an int array (the expert counts)
  int zero_n;
  // GEMM2 plain-row mode (expert parallelism): group row i goes to output row
  // c_row + i (or row i of the buffer at byte address group_base[g]), scaled
  // by row_w[c_row + i] (1 without row_w)
  int plain;
  const float* row_w;
  const unsigned long long* group_base;
  // BF16_OUT: out_bf16 [rows, out_ld] bf16, row c_row + i, columns < out_cols
  __nv_bfloat16* out_bf16;
  // SWIGLU_BWD (backward dz' = dh W_down; rows c_row + i, features < inter):
  // a | b in, g z, [da | db] and per-64-feature partials of <dz', z> out;
  // routed rows take their gate weight from row_w
  const __nv_bfloat16* ab;   // [rows, 2I]
  __nv_bfloat16* zg;         // [rows, I]
  __nv_bfloat16* dab;        // [rows, 2I]
  float* dgp;                // [rows, I / 64]
  // weight-gradient mode (template WG): group g contracts over K elements
  // kgroup[2g] .. + 128 kgroup[2g+1]; both operands carry one scale per row
  // and 128-element k-block, stored k-block-major: a_scale[kb][a_scale_ld],
  // b_scale[kb][b_scale_ld] (kb counted from K element 0); b_rows = rows of B
  const int* kgroup;
  int a_scale_ld, b_scale_ld, b_rows;
};

constexpr int SB_FLOATS = (NUM_EPI / 32) * 64;   // WG: per-warp column scales of a k-block
// Weight-gradient mode (WG) tiles are 128 x 128: each epilogue warp holds 32
// accumulator columns, which leaves it registers to spare, and stages its
// 32 rows x 64 bytes of bf16 output in shared memory.
constexpr int WG_BN = BN / 2;
constexpr int XOUT_BYTES = (NUM_EPI / 32) * 32 * (WG_BN / 4) * 2;

__host__ inline size_t smem_bytes(int stages, int n_groups, bool wg = false) {
  return 1024 + (size_t)stages * (BM * KB + (wg ? WG_BN : BN) * KB) +
         (wg ? (size_t)XOUT_BYTES : 0) +
         (size_t)(2 * stages + 14) * 8 + 16 + 2 * 4 * BM * sizeof(float) +
         SB_FLOATS * sizeof(float) + (size_t)(n_groups + 1) * 4 + (wg ? (size_t)n_groups * 16 : 0) +
         64;
}

// ----------------------------------------------------------------------------- shared pieces
// Promotion of one k-block partial into the warp's 64 accumulator columns:
// acc[0..31] += m0 * P[col0 .. col0+31], acc[32..63] += m1 * P[col0+32 ..],
// two batches of two 16-column TMEM loads (tb already points at col0).
__device__ __forceinline__ void promote64(uint32_t tb, float (&acc)[64], float m0, float m1) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t va[16], vb[16];
    tmem_ld16_nowait(tb + (uint32_t)(32 * h), va);
    tmem_ld16_nowait(tb + (uint32_t)(32 * h + 16), vb);
    tmem_wait_ld2(va, vb);
    const float m = h == 0 ? m0 : m1;
    const float2 mm = make_float2(m, m);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int o = 32 * h + 2 * i;
      const float2 r = __ffma2_rn(mm, make_float2(__uint_as_float(va[2 * i]),
                                                  __uint_as_float(va[2 * i + 1])),
                                  make_float2(acc[o], acc[o + 1]));
      acc[o] = r.x;
      acc[o + 1] = r.y;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int o = 32 * h + 16 + 2 * i;
      const float2 r = __ffma2_rn(mm, make_float2(__uint_as_float(vb[2 * i]),
                                                  __uint_as_float(vb[2 * i + 1])),
                                  make_float2(acc[o], acc[o + 1]));
      acc[o] = r.x;
      acc[o + 1] = r.y;
    }
  }
}

// Promotion with a scale per accumulator column (weight-gradient mode):
// acc[j] += (sa * sb[j]) * P[col0 + j], with sb the slice's NC column scales
// of this k-block in shared memory (every lane reads the same address).
template <int NC>
__device__ __forceinline__ void promote_cols(uint32_t tb, float (&acc)[NC], float sa,
                                             const float* sb) {
  const float2 a2 = make_float2(sa, sa);
#pragma unroll
  for (int h = 0; h < NC / 16; ++h) {
    float v[16];
    tmem_ld16(tb + (uint32_t)(16 * h), v);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int o = 16 * h + 2 * i;
      const float2 m = __fmul2_rn(a2, *reinterpret_cast<const float2*>(sb + o));
      const float2 r = __ffma2_rn(m, make_float2(v[2 * i], v[2 * i + 1]),
                                  make_float2(acc[o], acc[o + 1]));
      acc[o] = r.x;
      acc[o + 1] = r.y;
    }
  }
}

// 64 fp32 values as bf16 (round to nearest even) at dst, 16-byte stores.
__device__ __forceinline__ void store_bf16x64(__nv_bfloat16* dst, const float (&v)[64]) {
  uint4* o = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 8; ++j)
    o[j] = make_uint4(gemm::pack_bf16x2(v[8 * j], v[8 * j + 1]),
                      gemm::pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                      gemm::pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                      gemm::pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
}

// Backward epilogue of dz' = dh W_down for 64 features f0 .. f0+63 of row
// crow (gate weight gw, 1 for a shared expert): with a, b the pre-activations,
//   z = SiLU(a) b,  g z,  dz = g dz',  da = dz b SiLU'(a),  db = dz SiLU(a),
// and the partial <dz', z> over these features.  A padding row (valid false)
// gets zeros, so the weight-gradient quantisation may read it.
__device__ __forceinline__ void epi_swiglu_bwd(const float (&acc)[64], const Args& a,
                                               long long crow, int f0, float gw, bool valid) {
  const int I = a.inter;
  __nv_bfloat16* zr = a.zg + crow * I + f0;
  __nv_bfloat16* dar = a.dab + crow * 2 * I + f0;
  float dgs = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t wz[4], wa[4], wb[4];
    if (valid) {
      const uint4 ra = *reinterpret_cast<const uint4*>(a.ab + crow * 2 * I + f0 + 8 * c);
      const uint4 rb = *reinterpret_cast<const uint4*>(a.ab + crow * 2 * I + I + f0 + 8 * c);
      const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(&ra);
      const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(&rb);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float zz[2], da2[2], db2[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float av = h ? __high2float(ha[j]) : __low2float(ha[j]);
          const float bv = h ? __high2float(hb[j]) : __low2float(hb[j]);
          const float sg = 1.0f / (1.0f + __expf(-av));
          const float si = av * sg;
          const float z = si * bv;
          const float dzp = acc[8 * c + 2 * j + h];
          const float dz = gw * dzp;
          dgs = fmaf(dzp, z, dgs);
          zz[h] = gw * z;
          da2[h] = dz * bv * (sg * (1.0f + av * (1.0f - sg)));
          db2[h] = dz * si;
        }
        wz[j] = gemm::pack_bf16x2(zz[0], zz[1]);
        wa[j] = gemm::pack_bf16x2(da2[0], da2[1]);
        wb[j] = gemm::pack_bf16x2(db2[0], db2[1]);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) wz[j] = wa[j] = wb[j] = 0u;
    }
    reinterpret_cast<uint4*>(zr)[c] = make_uint4(wz[0], wz[1], wz[2], wz[3]);
    reinterpret_cast<uint4*>(dar)[c] = make_uint4(wa[0], wa[1], wa[2], wa[3]);
    reinterpret_cast<uint4*>(dar + I)[c] = make_uint4(wb[0], wb[1], wb[2], wb[3]);
  }
  a.dgp[crow * (I / 64) + f0 / 64] = valid ? dgs : 0.f;
}

// GEMM1 epilogue of one row's 64-column slice cs (gate columns 0..31, the
// matching up columns 32..63): H = SiLU(gate) * up, the row's 1x128 amax over
// the four slices through shared memory (xbar, bounded), E4M3 codes and the
// fp32 tile scale.  Returns false when the exchange wait gave up.
__device__ __forceinline__ bool epi_swiglu_q(float (&acc)[64], const Args& a, float* amax_buf,
                                             uint64_t* xbar, int tcount, int cs, int r, bool valid,
                                             size_t hrow, int nt, volatile int* abort_flag) {
  float pam = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    acc[i] = gemm::silu_f(acc[i]) * acc[32 + i];
    pam = fmaxf(pam, fabsf(acc[i]));
  }
  float* ab = amax_buf + (tcount & 1) * 4 * BM;
  ab[cs * BM + r] = pam;
  mbar_arrive(xbar);
  if (!mbar_wait(xbar, (uint32_t)tcount & 1u, abort_flag)) return false;
  const float amax = fmaxf(fmaxf(ab[r], ab[BM + r]), fmaxf(ab[2 * BM + r], ab[3 * BM + r]));
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 0.f;
  const float inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 0.f;
  if (valid) {
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      w[j] = (uint32_t)f32_to_e4m3(__fmul_rn(acc[4 * j], inv)) |
             ((uint32_t)f32_to_e4m3(__fmul_rn(acc[4 * j + 1], inv)) << 8) |
             ((uint32_t)f32_to_e4m3(__fmul_rn(acc[4 * j + 2], inv)) << 16) |
             ((uint32_t)f32_to_e4m3(__fmul_rn(acc[4 * j + 3], inv)) << 24);
    uint4* dst = reinterpret_cast<uint4*>(a.hq + hrow * a.inter + nt * 128 + cs * 32);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    if (cs == 0) a.hs[hrow * (a.inter / 128) + nt] = scale;
  }
  return true;
}

// GEMM2 epilogue of one row's 64 output columns (feature col): times the gate
// weight (1 for a shared expert) and written as bf16 to the row's slot, or in
// plain-row mode to the group's output row.
__device__ __forceinline__ void epi_scatter(const float (&acc)[64], const Args& a, int g,
                                            int grow, int col) {
  long long dst;
  float wgt = 1.0f;
  __nv_bfloat16* base = a.y;
  const int s_idx = a.gt.aux(g);
  if (a.plain) {
    const int crow = a.gt.c_row(g);
    if (a.group_base) {
      base = reinterpret_cast<__nv_bfloat16*>(a.group_base[g]);
      dst = grow;
    } else {
      dst = (long long)crow + grow;
    }
    wgt = a.row_w ? a.row_w[crow + grow] : 1.0f;
  } else if (s_idx < 0) {
    const int pair = a.pair_of[a.gt.c_row(g) + grow];
    const int t = pair / a.K, k = pair - t * a.K;
    dst = (long long)t * (a.K + a.Ks) + k;
    wgt = a.topk_w ? a.topk_w[pair] : 1.0f;   // the backward's du pieces carry no weight
  } else {
    dst = (long long)grow * (a.K + a.Ks) + a.K + s_idx;
  }
  uint4* o = reinterpret_cast<uint4*>(base + dst * a.d + col);
#pragma unroll
  for (int j = 0; j < 8; ++j)
    o[j] = make_uint4(gemm::pack_bf16x2(acc[8 * j] * wgt, acc[8 * j + 1] * wgt),
                      gemm::pack_bf16x2(acc[8 * j + 2] * wgt, acc[8 * j + 3] * wgt),
                      gemm::pack_bf16x2(acc[8 * j + 4] * wgt, acc[8 * j + 5] * wgt),
                      gemm::pack_bf16x2(acc[8 * j + 6] * wgt, acc[8 * j + 7] * wgt));
}

template <int KIND, int EPI, bool WG = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm_promoted(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, const Args a) {
  grid_dep_sync();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  constexpr int TBN = WG ? WG_BN : BN;     // accumulator columns of a tile
  // TMEM partials in flight: two of 256 columns, or four of 128 in the
  // weight-gradient mode, so its MMA runs further ahead of the promotion
  constexpr int NP = TMEM_COLS / TBN;
  constexpr int WC = TBN / 4;              // columns of one epilogue warp
  constexpr uint32_t a_bytes = BM * KB;
  constexpr uint32_t b_bytes = TBN * KB;
  constexpr uint32_t stage_bytes = a_bytes + b_bytes;
  const int S = a.stages;
  uint8_t* xout = smem + (size_t)S * stage_bytes;        // WG: 16 warps x 32 rows x 128 B
  uint64_t* full = reinterpret_cast<uint64_t*>(xout + (WG ? XOUT_BYTES : 0));
  uint64_t* empty = full + S;
  uint64_t* pfull = empty + S;
  uint64_t* pempty = pfull + NP;
  uint64_t* sfull = pempty + NP;     // WG: a partial slot's scales are in shared memory
  uint64_t* xbar = sfull + NP;       // amax exchange between the epilogue warps
  uint64_t* drain = xbar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* amax_buf = reinterpret_cast<float*>(tmem_slot + 4);   // [2][4][128]
  float* sb_buf = amax_buf + 2 * 4 * BM;   // WG: NP slots of BM row + TBN column scales
  int* s_prefix = reinterpret_cast<int*>(sb_buf + SB_FLOATS);
  int* s_kgroup = s_prefix + a.gt.count() + 1;                  // WG: the groups' K ranges

  const int warp = warp_id(), lane = lane_id();
  const int n_groups = a.gt.count();
  if (a.zero_ptr) {
    for (int i = blockIdx.x * NUM_THREADS + threadIdx.x; i < a.zero_n; i += gridDim.x * NUM_THREADS)
      a.zero_ptr[i] = 0;
  }
  for (int i = threadIdx.x; i <= n_groups; i += NUM_THREADS) s_prefix[i] = a.gt.prefix(i);
  if (WG)
    for (int i = threadIdx.x; i < n_groups; i += NUM_THREADS) {
      s_kgroup[4 * i] = a.kgroup[2 * i];
      s_kgroup[4 * i + 1] = a.kgroup[2 * i + 1];
      s_kgroup[4 * i + 2] = a.gt.c_row(i);
      s_kgroup[4 * i + 3] = a.gt.rows(i);
    }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int j = 0; j < NP; ++j) {
      mbar_init(&pfull[j], 1);
      mbar_init(&pempty[j], NUM_EPI / 32);
      mbar_init(&sfull[j], 1);
    }
    mbar_init(xbar, NUM_EPI);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
    }
    __syncwarp();
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = s_prefix[n_groups] * a.n_tiles_n;
  if (warp < EPI_WARP0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(CTRL_REGS));
    if (warp == 0) {
      // ------------------------------------------------------------------ TMA producer
      if (elect_one()) {
        int it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
          const int mt = tile / a.n_tiles_n, nt = tile - mt * a.n_tiles_n;
          const int g = gemm::find_group(s_prefix, n_groups, mt);
          const int lm = mt - s_prefix[g];
          const int arow = (a.a_from_crow ? a.gt.c_row(g) : a.gt.a_row(g)) + lm * BM;
          const int ebase = a.gt.expert(g) * a.b_rows_per_expert;
          const int k0 = WG ? s_kgroup[4 * g] : 0;
          const int nkb = WG ? s_kgroup[4 * g + 1] : a.num_kb;
          for (int kb = 0; kb < nkb; ++kb, ++it) {
            const int s = it % S;
            const uint32_t ph = (uint32_t)(it / S) & 1u;
            if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) { ok = false; break; }
            uint8_t* sa = smem + (size_t)s * stage_bytes;
            uint8_t* sb = sa + a_bytes;
            mbar_arrive_expect_tx(&full[s], stage_bytes);
            const int kx = k0 + kb * a.kb_elems;
            tma_load_2d(&tmA, &full[s], sa, kx, arow);
            if (EPI == EPI_SWIGLU_Q) {
              const int gr = ebase + nt * 128, ur = ebase + a.b_up_off + nt * 128;
  #pragma unroll
              for (int c = 0; c < 4; ++c) {
                tma_load_2d(&tmB, &full[s], sb + (size_t)(2 * c) * 32 * KB, kx, gr + 32 * c);
                tma_load_2d(&tmB, &full[s], sb + (size_t)(2 * c + 1) * 32 * KB, kx, ur + 32 * c);
              }
            } else {
              tma_load_2d(&tmB, &full[s], sb, kx, ebase + nt * TBN);
            }
          }
        }
        if (!ok) {
          volatile int no_abort = 0;
          for (int j = (it - S > 0 ? it - S : 0); j < it; ++j)
            mbar_wait(&full[j % S], (uint32_t)(j / S) & 1u, &no_abort);
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      if (elect_one()) {
        int it = 0, pu = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
          int nkb = a.num_kb;
          if (WG) {
            const int g = gemm::find_group(s_prefix, n_groups, tile / a.n_tiles_n);
            nkb = s_kgroup[4 * g + 1];
          }
          for (int kb = 0; kb < nkb; ++kb, ++it, ++pu) {
            const int s = it % S;
            const uint32_t ph = (uint32_t)(it / S) & 1u;
            const int p = pu % NP;
            const uint32_t pph = (uint32_t)(pu / NP) & 1u;
            if (!mbar_wait(&full[s], ph, abort_flag)) { ok = false; break; }
            if (!mbar_wait(&pempty[p], pph ^ 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + (size_t)s * stage_bytes);
            const uint64_t ad = umma_desc_sw128(sa);
            const uint64_t bd = umma_desc_sw128(sa + a_bytes);
            const uint32_t d_tmem = tmem_base + (uint32_t)(p * TBN);
  #pragma unroll
            for (int k = 0; k < KB / 32; ++k)
              umma<KIND>(d_tmem, ad + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), a.idesc,
                      k != 0 ? 1u : 0u);
            umma_commit(&empty[s]);
            umma_commit(&pfull[p]);
          }
        }
        // every MMA issued above completes before the block may free TMEM
        umma_commit(drain);
        volatile int no_abort = 0;
        mbar_wait(drain, 0, &no_abort);
      }
      __syncwarp();
    } else if (WG && warp == 2) {
      // ------------------------------------------------------------------ scale loader (WG)
      // the row and column scales of every (tile, k-block) into the shared
      // slot of its TMEM partial, up to NP k-blocks ahead of the promotion
      // (a slot is refilled once the promotion of its partial has released it)
      int pu = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        const int mt = tile / a.n_tiles_n, nt = tile - mt * a.n_tiles_n;
        const int g = gemm::find_group(s_prefix, n_groups, mt);
        const int* kg = s_kgroup + 4 * g;
        const int m0 = (mt - s_prefix[g]) * BM, n0 = nt * TBN;
        for (int kb = 0; kb < kg[1]; ++kb, ++pu) {
          const int p = pu % NP;
          if (!mbar_wait(&pempty[p], ((uint32_t)(pu / NP) & 1u) ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const size_t kr = (size_t)(kg[0] / 128 + kb);
          float* slot = sb_buf + p * (BM + TBN);
          // all eight loads in flight before the first store
          float v[(BM + TBN) / 32];
#pragma unroll
          for (int j = 0; j < BM / 32; ++j) {
            const int i = 32 * j + lane;
            v[j] = m0 + i < a.a_rows ? a.a_scale[kr * a.a_scale_ld + m0 + i] : 0.f;
          }
#pragma unroll
          for (int j = 0; j < TBN / 32; ++j) {
            const int i = 32 * j + lane;
            v[BM / 32 + j] = n0 + i < a.b_rows ? a.b_scale[kr * a.b_scale_ld + n0 + i] : 0.f;
          }
#pragma unroll
          for (int j = 0; j < (BM + TBN) / 32; ++j) slot[32 * j + lane] = v[j];
          __syncwarp();
          if (lane == 0) mbar_arrive(&sfull[p]);
        }
      }
      __syncwarp();
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(EPI_REGS));
    // ------------------------------------------------------------------ promotion + epilogue
    const int ew = warp - EPI_WARP0;
    const int q = warp & 3;
    const int cs = ew >> 2;                 // column slice 0..3 of WC columns
    const int r = q * 32 + lane;
    const int col0 = cs * WC;
    const int kb_blocks_b = a.b_rows_per_expert / 128;
    int pu = 0, tcount = 0;
    bool ok = true;
    if constexpr (WG) {
      // Weight gradients: short K ranges (an expert's rows), 128 x 128 tiles;
      // group data and the scales (staged by the scale-loader warp) come from
      // shared memory.
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++tcount) {
        const int mt = tile / a.n_tiles_n, nt = tile - mt * a.n_tiles_n;
        const int g = gemm::find_group(s_prefix, n_groups, mt);
        const int lm = mt - s_prefix[g];
        const int* kg = s_kgroup + 4 * g;           // k0, k-blocks, c_row, rows
        const int nkb = kg[1];
        const int ncol = nt * TBN + col0;
        float acc[WC];
#pragma unroll
        for (int i = 0; i < WC; ++i) acc[i] = 0.f;
        for (int kb = 0; kb < nkb; ++kb, ++pu) {
          const int p = pu % NP;
          const uint32_t par = (uint32_t)(pu / NP) & 1u;
          if (!mbar_wait(&sfull[p], par, abort_flag)) { ok = false; break; }
          const float* slot = sb_buf + p * (BM + TBN);
          const float sa_k = slot[r];
          if (!mbar_wait(&pfull[p], par, abort_flag)) { ok = false; break; }
          tc_fence_after();
          promote_cols<WC>(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(p * TBN + col0),
                           acc, sa_k, slot + BM + col0);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&pempty[p]);
        }
        if (!ok) break;
        if constexpr (EPI == EPI_BF16_OUT) {
          // stage the warp's 32 rows x 64 bytes (16-byte chunks XOR-swizzled
          // by row pair, no bank conflicts either way) and write them back 8
          // rows per instruction, 4 lanes a row
          static_assert(WC == 32, "staging layout assumes 32 columns a warp");
          uint8_t* xw = xout + (size_t)ew * 32 * 64;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(xw + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(gemm::pack_bf16x2(acc[8 * c], acc[8 * c + 1]),
                           gemm::pack_bf16x2(acc[8 * c + 2], acc[8 * c + 3]),
                           gemm::pack_bf16x2(acc[8 * c + 4], acc[8 * c + 5]),
                           gemm::pack_bf16x2(acc[8 * c + 6], acc[8 * c + 7]));
          __syncwarp();
          const int wrow0 = lm * BM + q * 32;       // the warp's first row in the group
          if (ncol + WC <= a.out_cols) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int rr = 8 * k + (lane >> 2), c = lane & 3;
              const uint4 v =
                  *reinterpret_cast<const uint4*>(xw + rr * 64 + ((c ^ ((rr >> 1) & 3)) << 4));
              if (wrow0 + rr < kg[3])
                *reinterpret_cast<uint4*>(a.out_bf16 + (size_t)(kg[2] + wrow0 + rr) * a.out_ld +
                                          ncol + c * 8) = v;
            }
          }
          __syncwarp();
        }
      }
    } else {
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++tcount) {
        const int mt = tile / a.n_tiles_n, nt = tile - mt * a.n_tiles_n;
        const int g = gemm::find_group(s_prefix, n_groups, mt);
        const int lm = mt - s_prefix[g];
        const int grow = lm * BM + r;
        const bool valid = grow < a.gt.rows(g);
        const int arow = (a.a_from_crow ? a.gt.c_row(g) : a.gt.a_row(g)) + grow;
        const size_t eb = (size_t)a.gt.expert(g) * kb_blocks_b;
        const float* sa_row = nullptr;
        const float* sb0 = nullptr;
        const float* sb1 = nullptr;
        if (EPI == EPI_F32_STORE) {
          // unscaled: plain fp32 accumulation of the k-block partials
        } else if (EPI == EPI_SWIGLU_Q) {
          sa_row = arow < a.a_rows ? a.a_scale + (size_t)arow * a.num_kb : nullptr;
          sb0 = a.b_scale + (eb + nt) * a.num_kb;                          // gate block
          sb1 = a.b_scale + (eb + a.b_up_off / 128 + nt) * a.num_kb;       // up block
        } else {
          sa_row = arow < a.a_rows ? a.a_scale + (size_t)arow * a.num_kb : nullptr;
          // a slice past the expert's last B row block (N not a multiple of 256)
          // is never stored; its scale read stays inside the expert's blocks
          sb0 = a.b_scale + (eb + min(2 * nt + cs / 2, kb_blocks_b - 1)) * a.num_kb;
          sb1 = sb0;
        }
        float acc[WC];
  #pragma unroll
        for (int i = 0; i < WC; ++i) acc[i] = 0.f;
        const bool scaled = EPI != EPI_F32_STORE;
        const int nkb = a.num_kb;
        const int ncol = nt * TBN + col0;
        float na = scaled ? (sa_row ? sa_row[0] : 0.f) : 1.f;
        float nb0 = scaled ? sb0[0] : 1.f, nb1 = scaled ? sb1[0] : 1.f;
        for (int kb = 0; kb < nkb; ++kb, ++pu) {
          const float m0 = na * nb0, m1 = na * nb1;
          if (scaled && kb + 1 < nkb) {
            na = sa_row ? sa_row[kb + 1] : 0.f;
            nb0 = sb0[kb + 1];
            nb1 = sb1[kb + 1];
          }
          const int p = pu % NP;
          if (!mbar_wait(&pfull[p], (uint32_t)(pu / NP) & 1u, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(p * TBN + col0);
          // the router's unscaled promotion is a paired FMA with multiplier 1
          promote64(tb, acc, m0, m1);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&pempty[p]);
        }
        if (!ok) break;
        if constexpr (EPI == EPI_F32_STORE) {
          if (valid) {
            float* orow = a.out + (size_t)(a.gt.c_row(g) + grow) * a.out_ld + nt * TBN + col0;
            const int c0 = nt * TBN + col0;
            if (c0 + 64 <= a.out_cols) {
  #pragma unroll
              for (int j = 0; j < 16; ++j)
                reinterpret_cast<float4*>(orow)[j] =
                    make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
            } else {
  #pragma unroll
              for (int j = 0; j < 64; ++j)
                if (c0 + j < a.out_cols) orow[j] = acc[j];
            }
          }
        } else if constexpr (EPI == EPI_SWIGLU_Q) {
          if (!epi_swiglu_q(acc, a, amax_buf, xbar, tcount, cs, r, valid,
                            (size_t)(a.gt.c_row(g) + grow), nt, abort_flag)) {
            ok = false;
            break;
          }
        } else if constexpr (EPI == EPI_BF16_OUT) {
          if (valid && ncol + 64 <= a.out_cols)
            store_bf16x64(a.out_bf16 + (size_t)(a.gt.c_row(g) + grow) * a.out_ld + ncol, acc);
        } else if constexpr (EPI == EPI_SWIGLU_BWD) {
          if (ncol + 64 <= a.inter) {
            const long long crow = (long long)a.gt.c_row(g) + grow;
            const float gw = (a.gt.aux(g) < 0 && valid) ? a.row_w[crow] : 1.0f;
            epi_swiglu_bwd(acc, a, crow, ncol, gw, valid);
          }
        } else {
          if (valid) epi_scatter(acc, a, g, grow, nt * TBN + col0);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace gemm8
}  // namespace moe
