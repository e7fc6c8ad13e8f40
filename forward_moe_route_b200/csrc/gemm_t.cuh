// Persistent grouped expert GEMM with weights on the UMMA M side and tokens
// on the N side (D^T = W X^T), on tcgen05 / TMEM, fed by TMA, run on CTA
// pairs (tcgen05.mma.cta_group::2).
//
// Used for the down projection (GEMM2).  A cluster of two CTAs (two SMs)
// computes a tile of 256 W_down rows (output features) x up to TN = 256
// tokens of one expert.  Each CTA loads its own 128 weight rows and half of
// the token tile into its shared memory; the UMMA issued by the even CTA (the
// leader) reads both CTAs' operands and writes each CTA's 128 rows x all
// tokens into that CTA's TMEM.  Per SM this moves 32 KB per 128-byte K step
// instead of 48 KB for a 1-SM 128 x 256 tile, for the same tensor-core work.
// The tile's UMMA takes the tile's own token count rounded up to 32, so an
// expert's last token tile wastes at most 31 columns of tensor-core work.
// The epilogue scales by each token's gate weight (1 for shared experts) and
// writes the features into the token's slot row.  Weight tiles run fastest
// inside an expert, so the clusters of one wave share the expert's token
// tiles in L2.
//
// Warp roles (384 threads, one CTA per SM, in both CTAs): warp 0 TMA
// producer, warp 1 MMA issuer (leader only), warp 2 TMEM allocator, warps
// 4..11 epilogue.  Epilogue warp w owns TMEM lanes 32*(w%4) .. +31 (32
// features) and every other 16-token chunk ((w-4)/4 selects the parity).  A
// chunk goes TMEM -> registers -> a per-warp shared-memory transpose ->
// 16-byte stores along the token's slot row.  Two accumulator buffers of 256
// TMEM columns each.
//
// Synchronisation:
//   full[s]   leader only: the leader's producer expects both CTAs' bytes; both
//             CTAs' TMA loads complete on it (cta_group::2 form, leader address)
//   empty[s]  both CTAs: the leader's MMA commits to its own and the peer's
//   tfull[a]  both CTAs: the leader's MMA commits to both after a tile
//   tempty[a] leader only: the epilogue threads of both CTAs arrive (the peer's
//             through its cluster address)
// Every wait is bounded; both CTAs finish with a cluster barrier before TMEM
// is freed, so no CTA leaves while its peer may still touch its barriers.
#pragma once

#include "common.cuh"
#include "gemm.cuh"

namespace moe {
namespace gemmt {

constexpr int WM = 128;            // weight rows per CTA (the pair covers 256)
constexpr int KB = 128;
constexpr int TN = 256;            // tokens per pair tile (128 per CTA)
constexpr int NUM_THREADS = 384;
constexpr int EPI_WARP0 = 4;
constexpr int NUM_EPI_WARPS = 8;
constexpr int XPOSE_BYTES = 16 * 32 * 4;
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 512;

struct Args {
  gemm::GroupTab gt;
  int n_wt;                // weight tiles of 256 rows per expert
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
  // plain-row mode (expert parallelism): group row i goes to output row
  // c_row + i, scaled by row_w[c_row + i] (1 without row_w); with group_base,
  // group g's row i goes to row i of the buffer at byte address group_base[g]
  // (which may be another GPU's memory: the expert outputs go straight back to
  // the ranks that sent the rows)
  int plain;
  const float* row_w;
  const unsigned long long* group_base;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap* map, uint32_t bar_cluster,
                                                 void* smem_dst, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"((uint64_t)map), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
template <int KIND>
__device__ __forceinline__ void umma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  if constexpr (KIND == 0) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}
// Arrive once on the barrier at `bar_cluster` (either CTA of the pair) when
// all tcgen05 operations issued so far have completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar_cluster)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}

__host__ inline size_t smem_bytes(int stages, int n_groups) {
  return 1024 + (size_t)stages * (WM * KB + (TN / 2) * KB) + (size_t)NUM_EPI_WARPS * XPOSE_BYTES +
         (size_t)(2 * stages + 5) * 8 + 16 + (size_t)(n_groups + 1) * 4 + 64;
}

template <int KIND>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_down_gemm(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmH,
                     const Args a) {
  grid_dep_sync();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  constexpr uint32_t a_bytes = WM * KB;
  constexpr uint32_t b_bytes = (TN / 2) * KB;
  constexpr uint32_t stage_bytes = a_bytes + b_bytes;
  const int S = a.stages;
  uint8_t* xpose = smem + (size_t)S * stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(xpose + NUM_EPI_WARPS * XPOSE_BYTES);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_prefix = reinterpret_cast<int*>(tmem_slot + 4);

  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int n_groups = a.gt.count();
  if (warp == 0) {
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
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmH);
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
  const int n_wt = a.n_wt;
  const int total_tiles = s_prefix[n_groups] * n_wt;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (elect_one()) {
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < total_tiles && ok; tile += n_pairs) {
        const int tt = tile / n_wt, wt = tile - tt * n_wt;
        const int g = gemm::find_group(s_prefix, n_groups, tt);
        const int tok0 = (tt - s_prefix[g]) * TN;
        const int ntok = min(TN, a.gt.rows(g) - tok0);
        const int nmma = (ntok + 31) & ~31;
        const int trow = a.gt.c_row(g) + tok0 + (int)rank * (nmma / 2);
        const int wrow = a.gt.expert(g) * a.w_rows_per_expert + wt * 2 * WM + (int)rank * WM;
        for (int kb = 0; kb < a.num_kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (uint32_t)(it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* sa = smem + (size_t)s * stage_bytes;
          const uint32_t full_leader = mapa(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * stage_bytes);
          const int kx = kb * a.kb_elems;
          tma_load_2d_pair(&tmW, full_leader, sa, kx, wrow);
          tma_load_2d_pair(&tmH, full_leader, sa + a_bytes, kx, trow);
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
        const int tt = tile / n_wt;
        const int g = gemm::find_group(s_prefix, n_groups, tt);
        const int tok0 = (tt - s_prefix[g]) * TN;
        const int ntok = min(TN, a.gt.rows(g) - tok0);
        const int nmma = (ntok + 31) & ~31;
        const uint32_t idesc = umma_idesc(a.fmt, 2 * WM, nmma);
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
            umma_pair<KIND>(d_tmem, wd + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), idesc,
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
    const int ew = warp - EPI_WARP0;
    const int q = warp & 3;
    const int par = ew >> 2;
    uint8_t* xb = xpose + (size_t)ew * XPOSE_BYTES;
    const bool bf = a.out_bf16 != 0;
    const uint32_t tempty_leader0 = mapa(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa(smem_u32(&tempty[1]), 0);
    int tcount = 0;
    for (int tile = pair; tile < total_tiles; tile += n_pairs, ++tcount) {
      const int tt = tile / n_wt, wt = tile - tt * n_wt;
      const int g = gemm::find_group(s_prefix, n_groups, tt);
      const int tok0 = (tt - s_prefix[g]) * TN;
      const int rows = a.gt.rows(g);
      const int ntok = min(TN, rows - tok0);
      const int acc = tcount & 1;
      const uint32_t use = (uint32_t)(tcount >> 1);
      if (!mbar_wait(&tfull[acc], use & 1u, abort_flag)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * ACC_COLS);
      const int fw0 = wt * 2 * WM + (int)rank * WM + q * 32;
      const int crow = a.gt.c_row(g);
      const int s_idx = a.gt.aux(g);
      const int nch = (ntok + 15) >> 4;
      uint8_t* ybase = a.group_base ? reinterpret_cast<uint8_t*>(a.group_base[g])
                                    : reinterpret_cast<uint8_t*>(a.y);
      long long dreg[8];
      float wreg[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int tok = tok0 + 32 * i + lane;
        dreg[i] = -1;
        wreg[i] = 0.f;
        if (32 * i < ntok && tok < rows) {
          if (a.plain) {
            dreg[i] = (a.group_base ? 0LL : (long long)crow) + tok;
            wreg[i] = a.row_w ? a.row_w[crow + tok] : 1.0f;
          } else if (s_idx < 0) {
            const int pr = a.pair_of[crow + tok];
            const int t = pr / a.K, k = pr - t * a.K;
            dreg[i] = (long long)t * (a.K + a.Ks) + k;
            wreg[i] = a.topk_w[pr];
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
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float w = __shfl_sync(0xffffffffu, wreg[(16 * c + j) >> 5], (16 * c + j) & 31);
            if (bf)
              reinterpret_cast<__nv_bfloat16*>(xb)[j * 32 + lane] = __float2bfloat16_rn(v[j] * w);
            else
              reinterpret_cast<float*>(xb)[j * 32 + lane] = v[j] * w;
          }
          __syncwarp();
          if (bf) {
#pragma unroll
            for (int m = 0; m < 2; ++m) {
              const int pi = lane + 32 * m, j = pi >> 2, pc = pi & 3;
              const long long dst =
                  __shfl_sync(0xffffffffu, dreg[(16 * c + 8 * m) >> 5], (16 * c + j) & 31);
              const uint4 val = *reinterpret_cast<const uint4*>(xb + j * 64 + pc * 16);
              const int feat = fw0 + pc * 8;
              if (dst >= 0 && feat < a.d)
                *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(ybase) +
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
                *reinterpret_cast<uint4*>(reinterpret_cast<float*>(ybase) + (size_t)dst * a.d +
                                          feat) = val;
            }
          }
          __syncwarp();
        }
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

}  // namespace gemmt
}  // namespace moe
