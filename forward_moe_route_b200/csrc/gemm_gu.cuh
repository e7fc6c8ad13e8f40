// Gate/up projection with the SwiGLU epilogue (GEMM1) on CTA pairs:
// H = SiLU(X W_gate^T) * (X W_up^T), weights on the UMMA M side and tokens on
// the N side (tcgen05.mma.cta_group::2).
//
// A cluster of two CTAs computes 128 H columns (expert features f0 .. f0+127)
// for up to TN = 256 tokens of one expert.  CTA r of the pair loads the 64
// W_gate rows f0+64r .. +63 and the matching 64 W_up rows as its 128 UMMA A
// rows, and half of the token tile as its share of B; the leader's M = 256
// UMMA writes each CTA's 128 rows x all tokens into that CTA's TMEM, so TMEM
// lanes 0-63 hold gate values and lanes 64-127 the up values of the same 64
// features.  Per SM a 128-byte K step moves 32 KB (a token-row tile of 128
// tokens x 256 gate/up columns moves 48 KB), and an expert's token tail is
// padded to a multiple of 32 tokens instead of 128.
//
// Epilogue (8 warps per CTA): warp w reads TMEM lane quadrant w % 4 and the
// 16-token chunks of parity (w - 4) / 4.  The up warps (quadrants 2, 3) copy
// their values into a shared exchange buffer; the gate warps (quadrants 0, 1)
// wait for it, form SiLU(gate) * up, transpose each 16-token chunk through a
// per-warp buffer and write 16-byte pieces of the token-major H rows.
//
// Synchronisation as in the pair down projection (full / empty / tfull /
// tempty, every wait bounded, a cluster barrier before TMEM is freed), plus
// xfull (the up warps' values are in the exchange buffer) and xempty (the
// gate warps have read them) once per tile.
//
// With Args::ab set the gate warps also write the rounded pre-activations
// a = X W_gate^T and the up warps b = X W_up^T of every row, so that a
// backward can skip recomputing them.
#pragma once

#include "common.cuh"
#include "gemm.cuh"
#include "gemm_t.cuh"

namespace moe {
namespace gemmgu {

constexpr int FM = 64;             // features per CTA (gate rows = up rows = FM)
constexpr int KB = 128;            // bytes of K per k-block
constexpr int TN = 256;            // tokens per pair tile (128 per CTA)
constexpr int NUM_THREADS = 384;
constexpr int EPI_WARP0 = 4;
constexpr int NUM_EPI_WARPS = 8;
constexpr int XPOSE_BYTES = 16 * 32 * 4;   // per gate warp: 16 tokens x 32 features (fp32)
constexpr int XCHG_BYTES = 2 * TN * 32 * 4; // up values: 2 quadrants x 256 tokens x 32 lanes
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 512;

struct Args {
  gemm::GroupTab gt;       // rows, a_row / a_map (token rows in x or x_perm), expert, c_row
  int n_ft;                // feature tiles of 128 per expert
  int num_kb;
  int kb_elems;
  int inter;               // I
  int w_rows_per_expert;   // 2I
  int stages;
  uint32_t fmt;            // UMMA operand format: 1 bf16, 2 tf32
  int out_bf16;
  void* h;                 // [rows, I]
  // optional [rows, 2I] bf16 copy of the pre-activations a | b (gate values
  // in columns 0..I-1, up values in I..2I-1), kept for the backward
  __nv_bfloat16* ab;
};

__host__ inline size_t smem_bytes(int stages, int n_groups) {
  return 1024 + (size_t)stages * (2 * FM * KB + (TN / 2) * KB) + XCHG_BYTES +
         (size_t)4 * XPOSE_BYTES + (size_t)(2 * stages + 7) * 8 + 16 +
         (size_t)(n_groups + 1) * 4 + 64;
}

template <int KIND>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gate_up_gemm(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const __grid_constant__ CUtensorMap tmXP, const Args a) {
  grid_dep_sync();
  using namespace gemmt;   // cluster helpers of the pair down projection
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  constexpr uint32_t half_a = FM * KB;                 // 64 gate (or up) rows
  constexpr uint32_t a_bytes = 2 * half_a;
  constexpr uint32_t b_bytes = (TN / 2) * KB;
  constexpr uint32_t stage_bytes = a_bytes + b_bytes;
  const int S = a.stages;
  float* xchg = reinterpret_cast<float*>(smem + (size_t)S * stage_bytes);
  uint8_t* xpose = reinterpret_cast<uint8_t*>(xchg) + XCHG_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(xpose + 4 * XPOSE_BYTES);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* xfull = tempty + 2;
  uint64_t* xempty = xfull + 1;
  uint64_t* drain = xempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_prefix = reinterpret_cast<int*>(tmem_slot + 4);

  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int n_groups = a.gt.count();
  if (warp == 0) {
    // token tiles of TN per group, exclusive prefix
    int carry = 0;
    for (int base = 0; base < n_groups; base += 32) {
      const int g = base + lane;
      const int v = g < n_groups ? (a.gt.rows(g) + TN - 1) / TN : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (g < n_groups) s_prefix[g] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_prefix[n_groups] = carry;
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&tfull[j], 1);
      mbar_init(&tempty[j], 2 * NUM_EPI_WARPS * 32);
    }
    mbar_init(xfull, 4);    // the four up warps, one arrival each
    mbar_init(xempty, 4);   // the four gate warps
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmXP);
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();      // barrier initialisation is visible to the peer from here on
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int n_ft = a.n_ft;
  const int total_tiles = s_prefix[n_groups] * n_ft;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (elect_one()) {
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < total_tiles && ok; tile += n_pairs) {
        const int tt = tile / n_ft, ft = tile - tt * n_ft;
        const int g = gemm::find_group(s_prefix, n_groups, tt);
        const int tok0 = (tt - s_prefix[g]) * TN;
        const int ntok = min(TN, a.gt.rows(g) - tok0);
        const int nmma = (ntok + 31) & ~31;
        const int trow = a.gt.a_row(g) + tok0 + (int)rank * (nmma / 2);
        const CUtensorMap* tB = a.gt.a_map(g) ? &tmXP : &tmX;
        const int grow = a.gt.expert(g) * a.w_rows_per_expert + ft * 2 * FM + (int)rank * FM;
        const int urow = grow + a.inter;
        for (int kb = 0; kb < a.num_kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (uint32_t)(it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* sa = smem + (size_t)s * stage_bytes;
          const uint32_t full_leader = mapa(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * stage_bytes);
          const int kx = kb * a.kb_elems;
          tma_load_2d_pair(&tmW, full_leader, sa, kx, grow);
          tma_load_2d_pair(&tmW, full_leader, sa + half_a, kx, urow);
          tma_load_2d_pair(tB, full_leader, sa + a_bytes, kx, trow);
        }
      }
      // the copies this CTA issued land before the block may leave (bounded)
      volatile int no_abort = 0;
      for (int j = (it - S > 0 ? it - S : 0); j < it; ++j)
        mbar_wait(&empty[j % S], (uint32_t)(j / S) & 1u, &no_abort);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader)
    if (leader && elect_one()) {
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = pair; tile < total_tiles && ok; tile += n_pairs, ++tcount) {
        const int tt = tile / n_ft;
        const int g = gemm::find_group(s_prefix, n_groups, tt);
        const int tok0 = (tt - s_prefix[g]) * TN;
        const int ntok = min(TN, a.gt.rows(g) - tok0);
        const int nmma = (ntok + 31) & ~31;
        const uint32_t idesc = umma_idesc(a.fmt, 2 * 2 * FM, nmma);
        const int acc = tcount & 1;
        const uint32_t use = (uint32_t)(tcount >> 1);
        if (!mbar_wait(&tempty[acc], (use & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * ACC_COLS);
        for (int kb = 0; kb < a.num_kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (uint32_t)(it / S) & 1u;
          if (!mbar_wait(&full[s], ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + (size_t)s * stage_bytes);
          const uint64_t ad = umma_desc_sw128(sa);
          const uint64_t bd = umma_desc_sw128(sa + a_bytes);
#pragma unroll
          for (int k = 0; k < KB / 32; ++k)
            umma_pair<KIND>(d_tmem, ad + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), idesc,
                            (kb | k) != 0 ? 1u : 0u);
          const uint32_t e_local = smem_u32(&empty[s]);
          umma_commit_pair(mapa(e_local, 0));
          umma_commit_pair(mapa(e_local, 1));
        }
        if (ok) {
          const uint32_t t_local = smem_u32(&tfull[acc]);
          umma_commit_pair(mapa(t_local, 0));
          umma_commit_pair(mapa(t_local, 1));
        }
      }
      umma_commit_pair(mapa(smem_u32(drain), 0));
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
    __syncwarp();
  } else if (warp >= EPI_WARP0) {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;                 // TMEM lane quadrant
    const int par = (warp - EPI_WARP0) >> 2;  // 16-token chunks of this parity
    const bool up_warp = q >= 2;
    const bool bf = a.out_bf16 != 0;
    float* xq = xchg + (size_t)(q & 1) * TN * 32;     // this quadrant pair's exchange rows
    uint8_t* xb = xpose + (size_t)((q & 1) * 2 + par) * XPOSE_BYTES;
    const uint32_t tempty_leader0 = mapa(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa(smem_u32(&tempty[1]), 0);
    int tcount = 0;
    for (int tile = pair; tile < total_tiles; tile += n_pairs, ++tcount) {
      const int tt = tile / n_ft, ft = tile - tt * n_ft;
      const int g = gemm::find_group(s_prefix, n_groups, tt);
      const int tok0 = (tt - s_prefix[g]) * TN;
      const int ntok = min(TN, a.gt.rows(g) - tok0);
      const int nch = (ntok + 15) >> 4;
      const int acc = tcount & 1;
      const uint32_t use = (uint32_t)(tcount >> 1);
      if (!mbar_wait(&tfull[acc], use & 1u, abort_flag)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * ACC_COLS);
      if (up_warp) {
        // the gate warps have read the previous tile's values
        if (!mbar_wait(xempty, ((uint32_t)tcount & 1u) ^ 1u, abort_flag)) break;
        // this warp's up features are those of gate quadrant q - 2
        const int f_up = ft * 2 * FM + (int)rank * FM + (q & 1) * 32 + lane;
        __nv_bfloat16* bsave =
            a.ab != nullptr && f_up < a.inter
                ? a.ab + ((size_t)a.gt.c_row(g) + tok0) * 2 * a.inter + a.inter + f_up
                : nullptr;
#pragma unroll 1
        for (int c = par; c < nch; c += 2) {
          float v[16];
          tmem_ld16(tb + (uint32_t)(16 * c), v);
#pragma unroll
          for (int j = 0; j < 16; ++j) xq[(16 * c + j) * 32 + lane] = v[j];
          if (bsave != nullptr) {
            // b of 16 tokens; each store writes 32 consecutive features of a row
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (16 * c + j < ntok)
                bsave[(size_t)(16 * c + j) * 2 * a.inter] = __float2bfloat16_rn(v[j]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(xfull);
      } else {
        if (!mbar_wait(xfull, (uint32_t)tcount & 1u, abort_flag)) break;
        const int f_warp = ft * 2 * FM + (int)rank * FM + q * 32;   // first feature of the warp
        const size_t hrow0 = (size_t)a.gt.c_row(g) + tok0;
#pragma unroll 1
        for (int c = par; c < nch; c += 2) {
          float v[16];
          tmem_ld16(tb + (uint32_t)(16 * c), v);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float h = gemm::silu_f(v[j]) * xq[(16 * c + j) * 32 + lane];
            if (bf)
              reinterpret_cast<__nv_bfloat16*>(xb)[j * 32 + lane] = __float2bfloat16_rn(h);
            else
              reinterpret_cast<float*>(xb)[j * 32 + lane] = h;
          }
          if (a.ab != nullptr && f_warp + lane < a.inter) {
            // a of 16 tokens (the up warps write b); lane = feature, so each
            // store writes 32 consecutive features of a row
            __nv_bfloat16* asave = a.ab + (hrow0 + 16 * c) * 2 * a.inter + f_warp + lane;
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (16 * c + j < ntok) asave[(size_t)j * 2 * a.inter] = __float2bfloat16_rn(v[j]);
          }
          __syncwarp();
          if (bf) {
            // token j: 32 features = 64 bytes = 4 pieces; 64 pieces, 2 per lane
#pragma unroll
            for (int m = 0; m < 2; ++m) {
              const int pi = lane + 32 * m, j = pi >> 2, pc = pi & 3;
              const int f = f_warp + pc * 8;
              if (16 * c + j < ntok && f < a.inter)
                *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.h) +
                                          (hrow0 + 16 * c + j) * a.inter + f) =
                    *reinterpret_cast<const uint4*>(xb + j * 64 + pc * 16);
            }
          } else {
            // token j: 32 features = 128 bytes = 8 pieces; 128 pieces, 4 per lane
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const int pi = lane + 32 * m, j = pi >> 3, pc = pi & 7;
              const int f = f_warp + pc * 4;
              if (16 * c + j < ntok && f < a.inter)
                *reinterpret_cast<uint4*>(reinterpret_cast<float*>(a.h) +
                                          (hrow0 + 16 * c + j) * a.inter + f) =
                    *reinterpret_cast<const uint4*>(xb + j * 128 + pc * 16);
            }
          }
          __syncwarp();
        }
        if (lane == 0) mbar_arrive(xempty);
      }
      tc_fence_before();
      if (leader) mbar_arrive(&tempty[acc]);
      else mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();      // the peer no longer touches this CTA's barriers or TMEM
  if (warp == 2) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

}  // namespace gemmgu
}  // namespace moe
