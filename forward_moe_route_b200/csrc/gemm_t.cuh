// Persistent grouped expert GEMM with weights on the UMMA M side and tokens
// on the N side (D^T = W X^T), on tcgen05 / TMEM, fed by TMA.
//
// Used for the down projection (GEMM2): a tile is 128 W_down rows (output
// features) x up to TN = 256 tokens of one expert.  The tile's UMMA takes the
// tile's own token count rounded up to 16, so an expert's last token tile
// wastes at most 15 rows of tensor-core work (a 128-row token tile would
// waste up to 127).  The epilogue scales by each token's gate weight (1 for
// shared experts) and writes the features into the token's slot row.
// The per-group token-tile prefix is computed by each CTA from the group table.
// Weight tiles run fastest inside an expert, so the CTAs of one wave share the
// expert's token tiles in L2 and each weight tile is reused across the
// expert's token tiles.
//
// Warp roles (384 threads, one CTA per SM): warp 0 TMA producer, warp 1 MMA
// issuer, warp 2 TMEM allocator, warps 4..11 epilogue.  Epilogue warp w owns
// TMEM lanes 32*(w%4) .. +31 (32 features) and every other 16-token chunk
// ((w-4)/4 selects the parity).  A chunk goes TMEM -> registers -> a per-warp
// shared-memory transpose -> 16-byte stores along the token's slot row.  Two
// accumulator buffers of 256 TMEM columns each.
#pragma once

#include "common.cuh"
#include "gemm.cuh"

namespace moe {
namespace gemmt {

constexpr int WM = 128;              // weight rows per tile (UMMA M)
constexpr int KB = 128;              // bytes of K per k-block
constexpr int NUM_THREADS = 384;
constexpr int EPI_WARP0 = 4;
constexpr int NUM_EPI_WARPS = 8;
constexpr int XPOSE_BYTES = 16 * 32 * 4;    // per-warp transpose buffer (16 tokens x 32 fp32)
constexpr int ACC_COLS = 256;        // TMEM columns per accumulator buffer
constexpr int TMEM_COLS = 512;


struct Args {
  gemm::GroupTab gt;
  int TN;                  // tokens per tile (256)
  int n_wt;                // weight tiles per expert (ceil(d/128))
  int num_kb;
  int kb_elems;
  int w_rows_per_expert;   // d
  int stages;
  uint32_t fmt;            // UMMA operand format: 1 bf16, 2 tf32
  int out_bf16;
  void* y;                 // [T*(K+Ks), d]
  int d;
  const int* pair_of;
  const float* topk_w;
  int K, Ks;
};

__host__ inline size_t smem_bytes(int a_bytes, int b_bytes, int stages, int n_groups) {
  return 1024 + (size_t)stages * (a_bytes + b_bytes) + (size_t)NUM_EPI_WARPS * XPOSE_BYTES +
         (size_t)(2 * stages + 5) * 8 + 16 + (size_t)(n_groups + 1) * 4 + 64;
}

template <int KIND>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_down_gemm(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmH,
                const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t a_bytes = WM * KB;
  const uint32_t b_bytes = (uint32_t)a.TN * KB;
  const uint32_t stage_bytes = a_bytes + b_bytes;
  const int S = a.stages;
  uint8_t* xpose = smem + (size_t)S * stage_bytes;   // NUM_EPI_WARPS x XPOSE_BYTES
  uint64_t* full = reinterpret_cast<uint64_t*>(xpose + NUM_EPI_WARPS * XPOSE_BYTES);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_prefix = reinterpret_cast<int*>(tmem_slot + 4);

  const int warp = warp_id(), lane = lane_id();
  const int n_groups = a.gt.count();
  // token-tile prefix over the groups: warp 0 scans ceil(rows / TN) 32 at a time
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < n_groups; base += 32) {
      const int g = base + lane;
      const int v = g < n_groups ? (a.gt.rows(g) + a.TN - 1) / a.TN : 0;
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
      mbar_init(&tempty[j], NUM_THREADS - EPI_WARP0 * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmH);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = s_prefix[n_groups] * a.n_wt;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (elect_one()) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        const int tt = tile / a.n_wt, wt = tile - tt * a.n_wt;
        const int g = gemm::find_group(s_prefix, n_groups, tt);
        const int tok0 = (tt - s_prefix[g]) * a.TN;
        const int trow = a.gt.c_row(g) + tok0;     // H rows of the group's tokens
        const int wrow = a.gt.expert(g) * a.w_rows_per_expert + wt * WM;
        for (int kb = 0; kb < a.num_kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (uint32_t)(it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* sa = smem + (size_t)s * stage_bytes;
          mbar_arrive_expect_tx(&full[s], stage_bytes);
          const int kx = kb * a.kb_elems;
          tma_load_2d(&tmW, &full[s], sa, kx, wrow);
          tma_load_2d(&tmH, &full[s], sa + a_bytes, kx, trow);
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
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++tcount) {
        const int tt = tile / a.n_wt;
        const int g = gemm::find_group(s_prefix, n_groups, tt);
        const int tok0 = (tt - s_prefix[g]) * a.TN;
        const int ntok = min(a.TN, a.gt.rows(g) - tok0);
        const int nmma = (ntok + 15) & ~15;
        const uint32_t idesc = umma_idesc(a.fmt, WM, nmma);
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
          const uint64_t wd = umma_desc_sw128(sa);
          const uint64_t bd = umma_desc_sw128(sa + a_bytes);
#pragma unroll
          for (int k = 0; k < KB / 32; ++k)
            umma<KIND>(d_tmem, wd + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), idesc,
                       (kb | k) != 0 ? 1u : 0u);
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&tfull[acc]);
      }
      umma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
    __syncwarp();
  } else if (warp >= EPI_WARP0) {
    // ------------------------------------------------------------------ epilogue
    const int ew = warp - EPI_WARP0;         // 0..7
    const int q = warp & 3;                  // TMEM lane quadrant: features q*32 .. +31
    const int par = ew >> 2;                 // this warp takes chunks c with c % 2 == par
    uint8_t* xb = xpose + (size_t)ew * XPOSE_BYTES;
    const bool bf = a.out_bf16 != 0;
    int tcount = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++tcount) {
      const int tt = tile / a.n_wt, wt = tile - tt * a.n_wt;
      const int g = gemm::find_group(s_prefix, n_groups, tt);
      const int tok0 = (tt - s_prefix[g]) * a.TN;
      const int rows = a.gt.rows(g);
      const int ntok = min(a.TN, rows - tok0);
      const int acc = tcount & 1;
      const uint32_t use = (uint32_t)(tcount >> 1);
      if (!mbar_wait(&tfull[acc], use & 1u, abort_flag)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * ACC_COLS);
      const int fw0 = wt * WM + q * 32;     // first feature of this warp
      const int crow = a.gt.c_row(g);
      const int s_idx = a.gt.aux(g);
      const int nch = (ntok + 15) >> 4;
      // slot row and gate weight of the tile's tokens: lane l holds those of
      // tokens l, l+32, ..., l+224; broadcast by shuffles
      long long dreg[8];
      float wreg[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int tok = tok0 + 32 * i + lane;
        dreg[i] = -1;
        wreg[i] = 0.f;
        if (32 * i < ntok && tok < rows) {
          if (s_idx < 0) {
            const int pair = a.pair_of[crow + tok];
            const int t = pair / a.K, k = pair - t * a.K;
            dreg[i] = (long long)t * (a.K + a.Ks) + k;
            wreg[i] = a.topk_w[pair];
          } else {
            dreg[i] = (long long)tok * (a.K + a.Ks) + a.K + s_idx;
            wreg[i] = 1.0f;
          }
        }
      }
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        if ((c & 1) == par && c < nch) {
          float v[16];
          tmem_ld16(tb + (uint32_t)(16 * c), v);
          // scale by each token's gate weight and transpose: xb[j][lane]
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float w = __shfl_sync(0xffffffffu, wreg[(16 * c + j) >> 5], (16 * c + j) & 31);
            if (bf)
              reinterpret_cast<__nv_bfloat16*>(xb)[j * 32 + lane] = __float2bfloat16_rn(v[j] * w);
            else
              reinterpret_cast<float*>(xb)[j * 32 + lane] = v[j] * w;
          }
          __syncwarp();
          // each token's 32 features leave as 16-byte pieces along its slot row
          if (bf) {
#pragma unroll
            for (int m = 0; m < 2; ++m) {
              const int pi = lane + 32 * m, j = pi >> 2, pc = pi & 3;
              const long long dst =
                  __shfl_sync(0xffffffffu, dreg[(16 * c + 8 * m) >> 5], (16 * c + j) & 31);
              const uint4 val = *reinterpret_cast<const uint4*>(xb + j * 64 + pc * 16);
              const int feat = fw0 + pc * 8;
              if (dst >= 0 && feat < a.d)
                *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.y) +
                                          (size_t)dst * a.d + feat) = val;
            }
          } else {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const int pi = lane + 32 * m, j = pi >> 3, pc = pi & 7;
              const long long dst =
                  __shfl_sync(0xffffffffu, dreg[(16 * c + 4 * m) >> 5], (16 * c + j) & 31);
              const uint4 val = *reinterpret_cast<const uint4*>(xb + j * 128 + pc * 16);
              const int feat = fw0 + pc * 4;
              if (dst >= 0 && feat < a.d)
                *reinterpret_cast<uint4*>(reinterpret_cast<float*>(a.y) + (size_t)dst * a.d +
                                          feat) = val;
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace gemmt
}  // namespace moe
