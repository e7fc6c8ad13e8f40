// Grouped GEMM of the layer backward: C_g = A_g B_g^T for a device-built list
// of problems, on tcgen05 / TMEM (the fp32 accumulator kept in TMEM over the
// whole K loop), fed by TMA, on clusters of two CTAs (tcgen05.mma.cta_group::2).
// Two kernels: k_gemm_bwd for the activation-side problems (A = token rows,
// K-major; 256-row tiles, each CTA loading its 128 rows and half of the
// tile's 256 B columns), and k_gemm_bwd_pair for the weight gradients (both
// operands MN-major, 256 x 256 tiles, fp32 output).
//
// Every backward GEMM contracts over an index that is the row index of one of
// its operands in memory: the hidden size d of W_down [d, I] (dz = dY W_down),
// the 2I rows of W_gu [2I, d] (du = [da | db] W_gu), and the expert's token
// rows for the weight gradients (dW_down = dY^T Z, dW_gu = [dA | dB]^T X).
// Instead of transposing those tensors in memory, an operand can be read
// "MN-major": the tile is loaded as 64-element (128-byte) slices of its M (or
// N) extent, one K row per 128-byte line with the 128-byte swizzle, and the
// UMMA instruction descriptor marks the operand as MN-major.  In the
// descriptor of such a tile, 8 K rows form a 1 KB core group (stride byte
// offset 1024) and consecutive 64-element slices are one TMA box apart
// (leading byte offset 64 rows x 128 bytes = 8 KB); one UMMA of K = 16 then
// starts 16 rows (2 KB) further on.  K-major operands use the same layout as
// the forward GEMMs.
//
// Problem table (int32, GB_FIELDS per problem), built on the device:
//   m, n, k            sizes (k may be 0: the tile is written as zeros)
//   a_map, a_m0, a_k0  which A tensor map and the problem's origin in it
//   b_map, b_n0, b_k0  the same for B
//   c_row0             first output row of the problem
//   m_pad              rows in [m, m_pad) of the output are written as zeros
//                      (row-store epilogues; the zero rows are the K padding
//                      of the weight-gradient GEMMs that read them later)
//   aux                epilogue-specific (shared-expert index or -1)
// Tiles: ceil(m/256) x ceil(n/256) per problem, N fastest, problems in
// order, strided over the persistent pairs.
//
// Warp roles (256 threads per CTA): warp 0 TMA producer, warp 1 MMA issuer
// (the even CTA's), warp 2 TMEM allocator, warps 4..7 epilogue (warp w reads
// TMEM lanes 32(w-4)..+31, one output row per thread).  Two accumulators of
// 256 columns.  full[s] on the leader receives both CTAs' bytes; the leader's
// MMA commits empty[s] and tfull[a] to both; both CTAs' epilogue threads
// arrive on the leader's tempty[a].  Every wait is bounded (see common.cuh),
// and a cluster barrier precedes the TMEM free.
#pragma once

#include "bulk.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "gemm_t.cuh"

namespace moe {
namespace gbwd {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;                 // bf16 elements per k-block (128 bytes)
constexpr int NUM_THREADS = 256;
constexpr int EPI_WARP0 = 4;
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 512;
constexpr int GB_FIELDS = 13;
constexpr uint32_t A_BYTES = BM * 128;
constexpr uint32_t B_BYTES = BN * 128;
constexpr uint32_t MN_BOX_BYTES = 64 * 128;   // one MN-major box: 64 K rows x 128 bytes

enum Epi {
  EPI_F32 = 0,          // C fp32 row-major (weight gradients)
  EPI_BF16 = 1,         // C bf16 row-major, rows [m, m_pad) zeroed
  EPI_SWIGLU_BWD = 2,   // dz' tile -> zg, [da | db], per-row <dz', z> partials
  EPI_SCATTER = 3       // bf16 rows to the token-major slots [T, K+Ks, d]
};

enum Field { F_M = 0, F_N, F_K, F_AMAP, F_AM0, F_AK0, F_BMAP, F_BN0, F_BK0, F_CROW, F_MPAD, F_AUX,
             F_SPARE };

struct Args {
  const int* tab;          // [n_probs][GB_FIELDS]
  int n_probs;
  int stages;
  void* c;                 // EPI_F32 / EPI_BF16 / EPI_SCATTER output
  long long ldc;           // elements per output row
  // EPI_SWIGLU_BWD
  const __nv_bfloat16* ab; // [rows, 2I] pre-activations a | b
  // pre-activations saved by the forward ([H rows, 2I], the forward's row
  // order; problem p's rows start at its F_SPARE field), read instead of ab
  const __nv_bfloat16* ab_saved;
  __nv_bfloat16* zg;       // [rows, I]  g * SiLU(a) * b
  __nv_bfloat16* dab;      // [rows, 2I] da | db
  float* dgp;              // [rows, I / 256] partial <dz', z>
  const float* row_w;      // [rows] gate weight of each padded row (routed problems)
  int inter;
  // EPI_SCATTER
  const int* row_pair;     // [rows] pair index t*K + k of each padded routed row (-1: pad)
  int K, Ks;
};

// Shared memory of k_gemm_bwd: a stage holds the CTA's 128 A rows and its
// half of the tile's 256 B columns.
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES / 2;
__host__ inline size_t smem_bytes(int stages, int n_probs) {
  return 1024 + (size_t)stages * STAGE_BYTES + (size_t)(2 * stages + 5) * 8 + 16 +
         (size_t)(n_probs + 1) * 4 + 64;
}

// UMMA descriptor of an MN-major operand tile loaded as 64-element boxes of
// 64 K rows each, 128-byte swizzle: core groups of 8 K rows (1 KB), boxes
// 8 KB apart along M / N.
__device__ __forceinline__ uint64_t umma_desc_sw128_mn(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFF) >> 4);
  d |= (uint64_t)(MN_BOX_BYTES >> 4) << 16;            // leading byte offset: next 64-element slice
  d |= (uint64_t)(1024 >> 4) << 32;                    // stride byte offset: next 8 K rows
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

template <bool B_MN, int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm_bwd(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
               const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
               const Args a) {
  static_assert(EPI != EPI_F32, "fp32 weight gradients run in k_gemm_bwd_pair");
  using namespace gemmt;   // cluster helpers of the forward pair kernels
  grid_dep_sync();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  constexpr int TM = 2 * BM;                          // rows per pair tile
  constexpr uint32_t SB = STAGE_BYTES;
  const int S = a.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * SB);
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
  const int np = a.n_probs;
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < np; base += 32) {
      const int g = base + lane;
      int v = 0;
      if (g < np) {
        const int* p = a.tab + (size_t)g * GB_FIELDS;
        v = ((p[F_M] + TM - 1) / TM) * ((p[F_N] + BN - 1) / BN);
      }
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (g < np) s_prefix[g] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_prefix[np] = carry;
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&tfull[j], 1);
      mbar_init(&tempty[j], 2 * 4 * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
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
  const int total = s_prefix[np];
  const int tile0 = (int)(blockIdx.x >> 1), tstep = (int)(gridDim.x >> 1);

  // tile -> (problem, m tile, n tile)
  auto locate = [&](int tile, int& g, int& mt, int& nt, const int*& p) {
    g = gemm::find_group(s_prefix, np, tile);
    p = a.tab + (size_t)g * GB_FIELDS;
    const int ntn = (p[F_N] + BN - 1) / BN;
    const int lt = tile - s_prefix[g];
    mt = lt / ntn;
    nt = lt - mt * ntn;
  };
  // the tile's UMMA N: its columns rounded up to 32, so each CTA's half of B
  // is a multiple of 16 columns
  auto mma_cols = [&](const int* p, int nt) {
    const int nc = min(BN, p[F_N] - nt * BN);
    return (nc + 31) & ~31;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (elect_one()) {
      int it = 0;
      bool ok = true;
      for (int tile = tile0; tile < total && ok; tile += tstep) {
        int g, mt, nt;
        const int* p;
        locate(tile, g, mt, nt, p);
        const int nkb = (p[F_K] + BK - 1) / BK;
        const CUtensorMap* tA = p[F_AMAP] ? &tmA1 : &tmA0;
        const CUtensorMap* tB = p[F_BMAP] ? &tmB1 : &tmB0;
        const int am = p[F_AM0] + mt * TM + (int)rank * BM, ak = p[F_AK0];
        const int bn = p[F_BN0] + nt * BN + (int)rank * (mma_cols(p, nt) / 2), bk = p[F_BK0];
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (uint32_t)(it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* sa = smem + (size_t)s * SB;
          uint8_t* sb = sa + A_BYTES;
          const int k0 = kb * BK;
          const uint32_t fl = mapa(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * SB);
          tma_load_2d_pair(tA, fl, sa, ak + k0, am);
          if (B_MN) {
            tma_load_2d_pair(tB, fl, sb, bn, bk + k0);
            tma_load_2d_pair(tB, fl, sb + MN_BOX_BYTES, bn + 64, bk + k0);
          } else {
            tma_load_2d_pair(tB, fl, sb, bk + k0, bn);
          }
        }
      }
      // the copies this CTA issued land before the block may leave (bounded)
      volatile int no_abort = 0;
      for (int j = (it - S > 0 ? it - S : 0); j < it; ++j)
        mbar_wait(&empty[j % S], (uint32_t)(j / S) & 1u, &no_abort);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (leader && elect_one()) {
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = tile0; tile < total && ok; tile += tstep, ++tcount) {
        int g, mt, nt;
        const int* p;
        locate(tile, g, mt, nt, p);
        const int nkb = (p[F_K] + BK - 1) / BK;
        const uint32_t idesc = umma_idesc(1, TM, mma_cols(p, nt)) | (B_MN ? (1u << 16) : 0u);
        const int acc = tcount & 1;
        const uint32_t use = (uint32_t)(tcount >> 1);
        if (!mbar_wait(&tempty[acc], (use & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * ACC_COLS);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (uint32_t)(it / S) & 1u;
          if (!mbar_wait(&full[s], ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + (size_t)s * SB);
          const uint64_t ad = umma_desc_sw128(sa);
          const uint64_t bd = B_MN ? umma_desc_sw128_mn(sa + A_BYTES) : umma_desc_sw128(sa + A_BYTES);
          // one UMMA per 16 elements of K: 32 bytes further along a K-major
          // line, 16 rows (2 KB) further down an MN-major tile
          constexpr uint64_t b_step = B_MN ? (2048 >> 4) : (32 >> 4);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint32_t accum = (kb | k) != 0 ? 1u : 0u;
            umma_pair<0>(d_tmem, ad + (uint64_t)(2 * k), bd + b_step * k, idesc, accum);
          }
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
    // ------------------------------------------------------------------ epilogue
    const int q = warp - EPI_WARP0;            // TMEM lane quadrant
    const int r_local = (int)rank * BM + q * 32 + lane;   // this thread's row of the tile
    const uint32_t tempty_leader0 = mapa(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa(smem_u32(&tempty[1]), 0);
    int tcount = 0;
    for (int tile = tile0; tile < total; tile += tstep, ++tcount) {
      int g, mt, nt;
      const int* p;
      locate(tile, g, mt, nt, p);
      const int acc = tcount & 1;
      const uint32_t use = (uint32_t)(tcount >> 1);
      if (!mbar_wait(&tfull[acc], use & 1u, abort_flag)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * ACC_COLS);
      const int m = p[F_M], n = p[F_N], mpad = p[F_MPAD];
      const int row = mt * TM + r_local;                  // row within the problem
      const bool has_k = p[F_K] > 0;
      const long long crow = (long long)p[F_CROW] + row;
      const int col0 = nt * BN;
      const int ncol = min(BN, n - col0);
      const bool valid = row < m;
      const bool zero_row = !valid && row < mpad;
      if (EPI == EPI_BF16 || EPI == EPI_SCATTER) {
        long long dst_row = crow;
        if (EPI == EPI_SCATTER && valid) {
          const int s_idx = p[F_AUX];
          if (s_idx < 0) {
            const int pr = a.row_pair[crow];
            dst_row = pr < 0 ? -1 : (long long)(pr / a.K) * (a.K + a.Ks) + pr % a.K;
          } else {
            dst_row = (long long)row * (a.K + a.Ks) + a.K + s_idx;
          }
        }
        const bool write = EPI == EPI_SCATTER ? (valid && dst_row >= 0) : (valid || zero_row);
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.c) + dst_row * a.ldc + col0;
#pragma unroll 1
        for (int c = 0; c < BN / 16; ++c) {
          float v[16];
          tmem_ld16(tb + (uint32_t)(16 * c), v);
          if (write && 16 * c < ncol) {
            const bool z = !valid || !has_k;
            uint32_t w[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
              w[j] = z ? 0u : gemm::pack_bf16x2(v[2 * j], v[2 * j + 1]);
            if (16 * c + 16 <= ncol) {
              reinterpret_cast<uint4*>(out + 16 * c)[0] = make_uint4(w[0], w[1], w[2], w[3]);
              reinterpret_cast<uint4*>(out + 16 * c)[1] = make_uint4(w[4], w[5], w[6], w[7]);
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (16 * c + j < ncol) out[16 * c + j] = __float2bfloat16_rn(z ? 0.f : v[j]);
            }
          }
        }
      } else {
        // EPI_SWIGLU_BWD: the tile holds dz' = dY W_down (unscaled) for 256
        // features of each row.  With a, b the forward pre-activations and g
        // the row's gate weight (1 for shared experts):
        //   z = SiLU(a) b,  zg = g z,  dz = g dz',
        //   da = dz b SiLU'(a),  db = dz SiLU(a),  dg partial = sum dz' z.
        const int I = a.inter;
        const float gw = (p[F_AUX] < 0 && valid) ? a.row_w[crow] : 1.0f;
        const __nv_bfloat16* abr =
            (a.ab_saved ? a.ab_saved + ((long long)p[F_SPARE] + row) * 2 * I : a.ab + crow * 2 * I) +
            col0;
        __nv_bfloat16* zr = a.zg + crow * I + col0;
        __nv_bfloat16* dar = a.dab + crow * 2 * I + col0;
        float dgs = 0.f;
#pragma unroll 1
        for (int c = 0; c < BN / 16; ++c) {
          float v[16];
          tmem_ld16(tb + (uint32_t)(16 * c), v);
          if ((valid || zero_row) && 16 * c < ncol) {
            uint32_t wz[8], wa[8], wb[8];
            if (valid && has_k) {
              const uint4* pa = reinterpret_cast<const uint4*>(abr + 16 * c);
              const uint4* pb = reinterpret_cast<const uint4*>(abr + I + 16 * c);
              uint4 ra[2] = {pa[0], pa[1]}, rb[2] = {pb[0], pb[1]};
              const __nv_bfloat162* ha = reinterpret_cast<const __nv_bfloat162*>(ra);
              const __nv_bfloat162* hb = reinterpret_cast<const __nv_bfloat162*>(rb);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                float zz[2], da2[2], db2[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const float av = h ? __high2float(ha[j]) : __low2float(ha[j]);
                  const float bv = h ? __high2float(hb[j]) : __low2float(hb[j]);
                  const float sg = 1.0f / (1.0f + __expf(-av));
                  const float si = av * sg;
                  const float z = si * bv;
                  const float dzp = v[2 * j + h];
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
              for (int j = 0; j < 8; ++j) wz[j] = wa[j] = wb[j] = 0u;
            }
            reinterpret_cast<uint4*>(zr + 16 * c)[0] = make_uint4(wz[0], wz[1], wz[2], wz[3]);
            reinterpret_cast<uint4*>(zr + 16 * c)[1] = make_uint4(wz[4], wz[5], wz[6], wz[7]);
            reinterpret_cast<uint4*>(dar + 16 * c)[0] = make_uint4(wa[0], wa[1], wa[2], wa[3]);
            reinterpret_cast<uint4*>(dar + 16 * c)[1] = make_uint4(wa[4], wa[5], wa[6], wa[7]);
            reinterpret_cast<uint4*>(dar + I + 16 * c)[0] = make_uint4(wb[0], wb[1], wb[2], wb[3]);
            reinterpret_cast<uint4*>(dar + I + 16 * c)[1] = make_uint4(wb[4], wb[5], wb[6], wb[7]);
          }
        }
        if (valid || zero_row) a.dgp[crow * ((I + BN - 1) / BN) + nt] = valid ? dgs : 0.f;
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

// ----------------------------------------------------------------------------- CTA pairs
// The weight-gradient problems (both operands MN-major, fp32 output) on CTA
// pairs: a cluster of two CTAs computes a 256 x 256 tile with one
// tcgen05.mma.cta_group::2 per K step issued by the even CTA; CTA r loads the
// A rows [256 mt + 128 r, +128) and the B columns of its half of the tile's N
// range, and its TMEM receives its 128 rows x the whole N.  Per SM a 64-row K
// step then moves 32 KB instead of 48 KB for the same tensor-core work: these
// GEMMs contract over one expert's rows only (~576 at the V3 shape), so the
// operand stream from L2, not the tensor pipe, sets their pace.
// Synchronisation as in the forward pair kernels (gemm_t.cuh): full[s] on the
// leader receives both CTAs' TMA bytes, the leader's MMA commits empty[s] and
// tfull[a] to both CTAs, both CTAs' epilogue threads arrive on the leader's
// tempty[a], every wait is bounded and a cluster barrier precedes the TMEM free.
constexpr int PBM = 256;                 // rows per pair tile (128 per CTA)
constexpr uint32_t PA_BYTES = 2 * MN_BOX_BYTES;   // a CTA's A: 128 rows of M (2 boxes of 64) x 64 K rows
constexpr uint32_t PB_BYTES = 2 * MN_BOX_BYTES;   // its half of B: up to 128 columns of N
constexpr uint32_t PSTAGE_BYTES = PA_BYTES + PB_BYTES;
// store staging: per epilogue warp two 32 x 32 blocks (4 KB each), written out
// by TMA: fp32 in the 128-byte-swizzled layout of the output tensor map, or
// bf16 (2 KB used) row-major for an unswizzled map
constexpr uint32_t PSTORE_BYTES = 4 * 2 * 4096;

__host__ inline size_t pair_smem_bytes(int stages, int n_probs) {
  return 1024 + (size_t)stages * PSTAGE_BYTES + PSTORE_BYTES + (size_t)(2 * stages + 5) * 8 + 16 +
         (size_t)(n_probs + 1) * 4 + 64;
}

// TMA store of one 32 x 32 fp32 block (the tensor map's box) from shared
// memory, completion tracked by the thread's bulk async-group.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* smem_src, int32_t x,
                                             int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          (uint64_t)map),
      "r"(smem_u32(smem_src)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

template <bool OUT_BF16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm_bwd_pair(const __grid_constant__ CUtensorMap tmA0,
                    const __grid_constant__ CUtensorMap tmA1,
                    const __grid_constant__ CUtensorMap tmB0,
                    const __grid_constant__ CUtensorMap tmB1,
                    const __grid_constant__ CUtensorMap tmC, const Args a) {
  using namespace gemmt;   // cluster helpers of the forward pair kernels
  grid_dep_sync();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int S = a.stages;
  uint8_t* store_buf = smem + (size_t)S * PSTAGE_BYTES;     // 1024-byte aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(store_buf + PSTORE_BYTES);
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
  const int np = a.n_probs;
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < np; base += 32) {
      const int g = base + lane;
      int v = 0;
      if (g < np) {
        const int* p = a.tab + (size_t)g * GB_FIELDS;
        v = ((p[F_M] + PBM - 1) / PBM) * ((p[F_N] + BN - 1) / BN);
      }
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (g < np) s_prefix[g] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_prefix[np] = carry;
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(&tfull[j], 1);
      mbar_init(&tempty[j], 2 * 4 * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmA1);
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
    tma_prefetch_desc(&tmC);
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
  const int total = s_prefix[np];
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  auto locate = [&](int tile, int& mt, int& nt, const int*& p) {
    const int g = gemm::find_group(s_prefix, np, tile);
    p = a.tab + (size_t)g * GB_FIELDS;
    const int ntn = (p[F_N] + BN - 1) / BN;
    const int lt = tile - s_prefix[g];
    mt = lt / ntn;
    nt = lt - mt * ntn;
  };
  // the tile's UMMA N (its columns rounded up to 32, so each CTA's half is a
  // multiple of 16 columns) and this CTA's first column
  auto tile_cols = [&](const int* p, int nt) {
    int nc = min(BN, p[F_N] - nt * BN);
    return (nc + 31) & ~31;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (elect_one()) {
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += n_pairs) {
        int mt, nt;
        const int* p;
        locate(tile, mt, nt, p);
        const int nkb = (p[F_K] + BK - 1) / BK;
        const CUtensorMap* tA = p[F_AMAP] ? &tmA1 : &tmA0;
        const CUtensorMap* tB = p[F_BMAP] ? &tmB1 : &tmB0;
        const int am = p[F_AM0] + mt * PBM + (int)rank * 128, ak = p[F_AK0];
        const int bn = p[F_BN0] + nt * BN + (int)rank * (tile_cols(p, nt) / 2), bk = p[F_BK0];
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (uint32_t)(it / S) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* sa = smem + (size_t)s * PSTAGE_BYTES;
          uint8_t* sb = sa + PA_BYTES;
          const uint32_t full_leader = mapa(smem_u32(&full[s]), 0);
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * PSTAGE_BYTES);
          const int k0 = ak + kb * BK, kb0 = bk + kb * BK;
          tma_load_2d_pair(tA, full_leader, sa, am, k0);
          tma_load_2d_pair(tA, full_leader, sa + MN_BOX_BYTES, am + 64, k0);
          tma_load_2d_pair(tB, full_leader, sb, bn, kb0);
          tma_load_2d_pair(tB, full_leader, sb + MN_BOX_BYTES, bn + 64, kb0);
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
      for (int tile = pair; tile < total && ok; tile += n_pairs, ++tcount) {
        int mt, nt;
        const int* p;
        locate(tile, mt, nt, p);
        const int nkb = (p[F_K] + BK - 1) / BK;
        const uint32_t idesc =
            umma_idesc(1, PBM, tile_cols(p, nt)) | (1u << 15) | (1u << 16);   // A, B MN-major
        const int acc = tcount & 1;
        const uint32_t use = (uint32_t)(tcount >> 1);
        if (!mbar_wait(&tempty[acc], (use & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * ACC_COLS);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (uint32_t)(it / S) & 1u;
          if (!mbar_wait(&full[s], ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + (size_t)s * PSTAGE_BYTES);
          const uint64_t ad = umma_desc_sw128_mn(sa);
          const uint64_t bd = umma_desc_sw128_mn(sa + PA_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_pair<0>(d_tmem, ad + (uint64_t)(128 * k), bd + (uint64_t)(128 * k), idesc,
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
    // Warp q owns TMEM lanes 32q .. 32q+31 (output rows); per 32-column chunk
    // it writes the block into one of its two swizzled staging buffers and
    // one lane stores it with TMA.  The output map's rows are one expert's
    // (m) and its columns the full row (N = ldc), so the store clips the
    // tile's edges itself.
    const int q = warp - EPI_WARP0;
    uint8_t* stg = store_buf + (size_t)q * 2 * 4096;
    const uint32_t tempty_leader0 = mapa(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa(smem_u32(&tempty[1]), 0);
    int tcount = 0, nst = 0;
    for (int tile = pair; tile < total; tile += n_pairs, ++tcount) {
      int mt, nt;
      const int* p;
      locate(tile, mt, nt, p);
      const int acc = tcount & 1;
      const uint32_t use = (uint32_t)(tcount >> 1);
      if (!mbar_wait(&tfull[acc], use & 1u, abort_flag)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * ACC_COLS);
      const int m = p[F_M];
      const bool has_k = p[F_K] > 0;
      const int col0 = nt * BN;
      const int nc = (min(BN, p[F_N] - col0) + 31) >> 5;    // 32-column chunks with data
      const int row0 = mt * PBM + (int)rank * 128 + q * 32;  // first row (within m) of the warp
      const int z = m > 0 ? p[F_CROW] / m : 0;
      const int nchunks = row0 < m ? nc : 0;
      if (nchunks == 0) {
        tc_fence_before();
        if (leader) mbar_arrive(&tempty[acc]);
        else mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
        continue;
      }
#pragma unroll 1
      for (int c = 0; c < nchunks; ++c, ++nst) {
        uint32_t va[16], vb[16];
        tmem_ld16_nowait(tb + (uint32_t)(32 * c), va);
        tmem_ld16_nowait(tb + (uint32_t)(32 * c + 16), vb);
        tmem_wait_ld2(va, vb);
        if (c == nchunks - 1) {
          // the warp's last TMEM read of the tile: hand the accumulator back
          tc_fence_before();
          if (leader) mbar_arrive(&tempty[acc]);
          else mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
        }
        uint8_t* buf = stg + (size_t)(nst & 1) * 4096;
        // the store issued from this buffer two chunks ago has read it
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        if (OUT_BF16) {
          // row `lane`: 32 bf16 = 64 bytes, plain row-major (the map has no swizzle)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t* src = j < 2 ? &va[8 * j] : &vb[8 * (j - 2)];
            uint32_t w4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              w4[i] = has_k ? gemm::pack_bf16x2(__uint_as_float(src[2 * i]),
                                                __uint_as_float(src[2 * i + 1]))
                            : 0u;
            *reinterpret_cast<uint4*>(buf + lane * 64 + j * 16) =
                make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        } else {
          // row `lane`, 16-byte piece j at (j ^ (row % 8)) (128-byte swizzle)
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t* src = j < 4 ? &va[4 * j] : &vb[4 * (j - 4)];
            const uint4 v = has_k ? make_uint4(src[0], src[1], src[2], src[3])
                                  : make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) = v;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tmC, buf, col0 + 32 * c, row0, z);
          bulk_commit_group();
        }
      }
    }
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
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

}  // namespace gbwd
}  // namespace moe
