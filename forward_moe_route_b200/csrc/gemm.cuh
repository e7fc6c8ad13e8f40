// Persistent grouped GEMM on tcgen05 / TMEM, fed by TMA: the gate/up
// projection with the SwiGLU epilogue (GEMM1).
//
// One launch computes C_g = A_g * B_g^T for a list of row groups g (one per
// expert), each A_g a block of token rows and B_g one expert's W_gate / W_up
// rows, both K-major.  The output tile is
// 128 rows x bn accumulator columns; tiles are numbered n-fastest across all
// groups and strided over the persistent CTAs.
//
// Warp roles (256 threads, one CTA per SM):
//   warp 0      TMA producer: A tile (128 x 128 B) + B tile (bn x 128 B) per stage
//   warp 1      MMA issuer: 4 UMMAs (K = 32 bytes each) per stage, accumulator in TMEM
//   warp 2      TMEM allocator
//   warps 4..7  epilogue: tcgen05.ld of one accumulator row per thread, fused
//               math, direct 16-byte stores
// Two TMEM accumulators let the epilogue of tile i overlap the MMAs of tile
// i+1.  Every wait is bounded (see mbar_wait).
#pragma once

#include "common.cuh"

namespace moe {
namespace gemm {

constexpr int BM = 128;            // tile rows = UMMA M (cta_group::1)
constexpr int KB = 128;            // bytes of K per stage = one 128-byte swizzle row
constexpr int NUM_THREADS = 256;
constexpr int EPI_WARP0 = 4;

enum Epi { EPI_SWIGLU = 1 };

// Group table (device, int32), struct of arrays for n groups:
//   [0, n]           m-tile prefix (exclusive scan of ceil(rows/128)), n+1 entries
//   rows[n]          valid rows of the group
//   a_row[n]         first row of the group in the A tensor map
//   a_map[n]         which A tensor map (0 or 1)
//   expert[n]        expert index (selects the B rows)
//   c_row[n]         first output row (GEMM1: H row; GEMM2: the group's H row)
//   aux[n]           -1 for routed groups, shared-expert index s otherwise
// With base == nullptr the table is one group of `single_rows` rows starting
// at row 0 of everything (the router GEMM).
struct GroupTab {
  const int* base;
  int n;
  int single_rows;
  __device__ __forceinline__ int count() const { return base ? n : 1; }
  __device__ __forceinline__ int prefix(int i) const {
    return base ? base[i] : (i == 0 ? 0 : (single_rows + 127) / 128);
  }
  __device__ __forceinline__ int rows(int g) const { return base ? base[n + 1 + g] : single_rows; }
  __device__ __forceinline__ int a_row(int g) const { return base ? base[n + 1 + n + g] : 0; }
  __device__ __forceinline__ int a_map(int g) const { return base ? base[n + 1 + 2 * n + g] : 0; }
  __device__ __forceinline__ int expert(int g) const { return base ? base[n + 1 + 3 * n + g] : 0; }
  __device__ __forceinline__ int c_row(int g) const { return base ? base[n + 1 + 4 * n + g] : 0; }
  __device__ __forceinline__ int aux(int g) const { return base ? base[n + 1 + 5 * n + g] : -1; }
};
__host__ __device__ constexpr int group_tab_ints(int n) { return n + 1 + 6 * n; }

struct Args {
  GroupTab gt;
  int n_tiles_n;       // tiles along N
  int num_kb;          // k-blocks (128 bytes of K each)
  int kb_elems;        // elements per k-block (64 bf16, 32 fp32)
  int bn;              // accumulator columns per tile (UMMA N)
  int b_half;          // SWIGLU: rows per half tile (gate / up); else 0
  int b_up_off;        // SWIGLU: row offset of W_up inside an expert (I)
  int b_rows_per_expert;
  int a_from_crow;     // A rows come from c_row (GEMM2 reads H)
  int stages;
  uint32_t idesc;
  uint32_t tmem_cols;
  // epilogue
  void* out;
  long long out_ld;    // elements per output row
  int out_bf16;        // 1: bf16 output, 0: fp32
};

__device__ __forceinline__ int find_group(const int* prefix, int n, int mt) {
  int lo = 0, hi = n;  // prefix[lo] <= mt < prefix[hi]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (prefix[mid] <= mt) lo = mid; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Store 16 consecutive fp32 values as bf16 (32 bytes) or fp32 (64 bytes).
__device__ __forceinline__ void store16(void* dst, const float (&v)[16], int bf16) {
  if (bf16) {
    uint4* p = reinterpret_cast<uint4*>(dst);
    p[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                      pack_bf16x2(v[6], v[7]));
    p[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                      pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
  } else {
    float4* p = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

template <int KIND, int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_grouped_gemm(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                   const __grid_constant__ CUtensorMap tmB, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t a_bytes = BM * KB;
  const uint32_t b_bytes = (uint32_t)a.bn * KB;
  const uint32_t stage_bytes = a_bytes + b_bytes;
  const int S = a.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * stage_bytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_prefix = reinterpret_cast<int*>(tmem_slot + 4);

  const int warp = warp_id(), lane = lane_id();
  const int n_groups = a.gt.count();

  for (int i = threadIdx.x; i <= n_groups; i += NUM_THREADS) s_prefix[i] = a.gt.prefix(i);
  if (threadIdx.x == 0) {
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
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, a.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int total_tiles = s_prefix[n_groups] * a.n_tiles_n;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (elect_one()) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        const int mt = tile / a.n_tiles_n, nt = tile - mt * a.n_tiles_n;
        const int g = find_group(s_prefix, n_groups, mt);
        const int lm = mt - s_prefix[g];
        const int arow = (a.a_from_crow ? a.gt.c_row(g) : a.gt.a_row(g)) + lm * BM;
        const CUtensorMap* tA = (!a.a_from_crow && a.gt.a_map(g)) ? &tmA1 : &tmA0;
        const int ebase = a.gt.expert(g) * a.b_rows_per_expert;
        const int brow = ebase + nt * (EPI == EPI_SWIGLU ? a.b_half : a.bn);
        for (int kb = 0; kb < a.num_kb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (uint32_t)(it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* sa = smem + (size_t)s * stage_bytes;
          uint8_t* sb = sa + a_bytes;
          mbar_arrive_expect_tx(&full[s], stage_bytes);
          const int kx = kb * a.kb_elems;
          tma_load_2d(tA, &full[s], sa, kx, arow);
          if (EPI == EPI_SWIGLU) {
            tma_load_2d(&tmB, &full[s], sb, kx, brow);
            tma_load_2d(&tmB, &full[s], sb + (size_t)a.b_half * KB, kx, brow + a.b_up_off);
          } else {
            tma_load_2d(&tmB, &full[s], sb, kx, brow);
          }
        }
      }
      if (!ok) {
        // Aborted: let the copies already issued land before the CTA exits.
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
        const int acc = tcount & 1;
        const uint32_t use = (uint32_t)(tcount >> 1);
        if (!mbar_wait(&tempty[acc], (use & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)acc * (a.tmem_cols / 2);
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
            umma<KIND>(d_tmem, ad + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), a.idesc,
                       (kb | k) != 0 ? 1u : 0u);
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&tfull[acc]);
      }
      // Every MMA issued above completes before the block may free TMEM.
      umma_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort);
    }
    __syncwarp();
  } else if (warp >= EPI_WARP0) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;             // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;        // tile row owned by this thread
    int tcount = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++tcount) {
      const int mt = tile / a.n_tiles_n, nt = tile - mt * a.n_tiles_n;
      const int g = find_group(s_prefix, n_groups, mt);
      const int lm = mt - s_prefix[g];
      const int acc = tcount & 1;
      const uint32_t use = (uint32_t)(tcount >> 1);
      if (!mbar_wait(&tfull[acc], use & 1u, abort_flag)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * (a.tmem_cols / 2);
      const int grow = lm * BM + r;                 // row inside the group
      const bool valid = grow < a.gt.rows(g);
      {
        const int hn = a.b_half;
        const size_t esz = a.out_bf16 ? 2 : 4;
        uint8_t* orow = reinterpret_cast<uint8_t*>(a.out) +
                        ((size_t)(a.gt.c_row(g) + grow) * (size_t)a.out_ld + (size_t)nt * hn) * esz;
        for (int c = 0; c < hn; c += 16) {
          float gv[16], uv[16];
          tmem_ld16(tb + (uint32_t)c, gv);
          tmem_ld16(tb + (uint32_t)(hn + c), uv);
#pragma unroll
          for (int i = 0; i < 16; ++i) gv[i] = silu_f(gv[i]) * uv[i];
          if (valid) store16(orow + (size_t)c * esz, gv, a.out_bf16);
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
    tmem_dealloc(tmem_base, a.tmem_cols);
  }
}

// Shared memory a launch needs for `stages` stages of a bn-column tile.
__host__ inline size_t smem_bytes(int bn, int stages, int n_groups) {
  size_t stage = (size_t)BM * KB + (size_t)bn * KB;
  return 1024 + (size_t)stages * stage + (size_t)(2 * stages + 5) * 8 + 16 +
         (size_t)(n_groups + 1) * 4 + 64;
}

}  // namespace gemm
}  // namespace moe
