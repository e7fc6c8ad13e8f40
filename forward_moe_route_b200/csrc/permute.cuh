// Token -> expert permutation, expert-contiguous gather (with fused 1x128 E4M3
// quantisation), group-table preparation for the grouped GEMMs, and the
// weighted combine.
//
// Permutation: the pair (t, k) with expert e = idx[t,k] goes to row
// offsets[e] + #{t' < t : e in idx[t']}.  It is built deterministically from
// per-chunk histograms (chunks of CHUNK tokens), a scan over chunks and
// experts, and an in-order walk of each chunk, so it is stable by token and
// identical from run to run.
#pragma once

#include <type_traits>

#include "bulk.cuh"
#include "common.cuh"
#include "gemm.cuh"

namespace moe {
namespace perm {

constexpr int CHUNK = 128;  // tokens per histogram chunk

// hist[c * N + e] = number of pairs of chunk c routed to expert e.
__global__ void __launch_bounds__(256) k_hist(const int32_t* __restrict__ idx, int T, int K, int N,
                                              int32_t* __restrict__ hist) {
  grid_dep_sync();
  extern __shared__ int32_t sh[];
  for (int e = threadIdx.x; e < N; e += blockDim.x) sh[e] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * CHUNK;
  const int t1 = min(T, t0 + CHUNK);
  for (int i = t0 * K + threadIdx.x; i < t1 * K; i += blockDim.x) {
    const int e = idx[i];
    if ((unsigned)e < (unsigned)N) atomicAdd(&sh[e], 1);
    else set_status(MOE_ERR_DEVICE_CHECK);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < N; e += blockDim.x) hist[(size_t)blockIdx.x * N + e] = sh[e];
}

// One block of 1024 threads.  Turns hist into each chunk's first row per
// expert (offsets[e] + pairs of expert e in earlier chunks), writes offsets
// [N+1], and checks the per-expert totals against `counts` (when given) or
// writes them to `counts_out` (when given).
//
// Thread (q, part) owns experts 4q..4q+3 (16-byte loads along a histogram row;
// N % 4 == 0, else one expert per thread) and a contiguous run of chunks; runs
// of up to SCAN_REG chunks stay in registers, so the histogram is read once
// and written once.
constexpr int SCAN_REG = 8;

template <int V>
__global__ void __launch_bounds__(1024) k_scan(int32_t* __restrict__ hist, int n_chunks, int N,
                                               const int32_t* __restrict__ counts,
                                               int32_t* __restrict__ counts_out,
                                               int32_t* __restrict__ offsets) {
  grid_dep_sync();
  __shared__ int32_t part_sum[1024 * V];   // [part][expert]
  __shared__ int32_t tot[512];
  __shared__ int32_t warp_tot[32];
  using vec_t = typename std::conditional<V == 4, int4, int>::type;
  const int groups = (N + V - 1) / V;                      // expert groups of V
  // parts per group: as many as the threads allow, but each part covers at
  // least 4 chunks, since the totals and the part prefix walk the parts serially
  const int P = max(1, min((int)(blockDim.x / groups), (n_chunks + 3) / 4));
  const int tid = threadIdx.x;
  const int q = tid % groups, part = tid / groups;
  const bool active = part < P && tid < groups * P;
  const int per = (n_chunks + P - 1) / P;
  const int c0 = part * per, c1 = min(n_chunks, c0 + per);
  auto load = [&](int c) -> vec_t { return *reinterpret_cast<const vec_t*>(hist + (size_t)c * N + q * V); };
  auto store = [&](int c, vec_t v) { *reinterpret_cast<vec_t*>(hist + (size_t)c * N + q * V) = v; };
  auto lane_of = [&](const vec_t& v, int i) -> int {
    if constexpr (V == 4) return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
    else return v;
  };
  vec_t reg[SCAN_REG];
  const bool in_regs = c1 - c0 <= SCAN_REG;
  int sum[V];
#pragma unroll
  for (int i = 0; i < V; ++i) sum[i] = 0;
  if (active) {
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < SCAN_REG; ++j)
        if (c0 + j < c1) reg[j] = load(c0 + j);
#pragma unroll
      for (int j = 0; j < SCAN_REG; ++j)
        if (c0 + j < c1) {
#pragma unroll
          for (int i = 0; i < V; ++i) sum[i] += lane_of(reg[j], i);
        }
    } else {
#pragma unroll 8
      for (int c = c0; c < c1; ++c) {
        const vec_t v = load(c);
#pragma unroll
        for (int i = 0; i < V; ++i) sum[i] += lane_of(v, i);
      }
    }
#pragma unroll
    for (int i = 0; i < V; ++i) part_sum[part * groups * V + q * V + i] = sum[i];
  }
  __syncthreads();
  // expert totals (parts in order) and the check against counts
  for (int e = tid; e < N; e += blockDim.x) {
    int total = 0;
    for (int pp = 0; pp < P; ++pp) total += part_sum[pp * groups * V + e];
    tot[e] = total;
    if (counts && counts[e] != total) set_status(MOE_ERR_DEVICE_CHECK);
    if (counts_out) counts_out[e] = total;
  }
  __syncthreads();
  // exclusive scan of tot[0..N) -> offsets (N <= 512: two elements a thread at most)
  const int v0 = tid < N ? tot[tid] : 0;
  int incl = v0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane_id() >= o) incl += y;
  }
  if (lane_id() == 31) warp_tot[warp_id()] = incl;
  __syncthreads();
  if (warp_id() == 0) {
    const int wv = warp_tot[lane_id()];
    int wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane_id() >= o) wi += y;
    }
    warp_tot[lane_id()] = wi - wv;
  }
  __syncthreads();
  const int excl = incl - v0 + warp_tot[warp_id()];
  __syncthreads();
  if (tid < N) {
    offsets[tid] = excl;
    if (tid == N - 1) offsets[N] = excl + v0;
    tot[tid] = excl;                       // now the expert's first row
  }
  __syncthreads();
  // each part's first row per expert: the expert base plus the earlier parts
  if (active) {
    int run[V];
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const int e = q * V + i;
      int r = e < N ? tot[e] : 0;
      for (int pp = 0; pp < part; ++pp) r += part_sum[pp * groups * V + e];
      run[i] = r;
    }
    auto emit = [&](int c, const vec_t& h) {
      vec_t o;
      if constexpr (V == 4) {
        o.x = run[0]; o.y = run[1]; o.z = run[2]; o.w = run[3];
        run[0] += h.x; run[1] += h.y; run[2] += h.z; run[3] += h.w;
      } else {
        o = run[0];
        run[0] += h;
      }
      store(c, o);
    };
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < SCAN_REG; ++j)
        if (c0 + j < c1) emit(c0 + j, reg[j]);
    } else {
#pragma unroll 8
      for (int c = c0; c < c1; ++c) emit(c, load(c));
    }
  }
}

// One block of SLOT_WARPS warps per chunk.  Warp w owns tokens
// [16w, 16w+16) of the chunk: it first counts its pairs per expert, a prefix
// over the warps gives each warp its first row per expert, and then each warp
// walks its tokens in order handing out rows (distinct experts within a token
// never collide), so the result is the same stable order as a single walk.
constexpr int SLOT_WARPS = 8;
constexpr int SLOT_TOKENS = CHUNK / SLOT_WARPS;   // 16

__global__ void __launch_bounds__(SLOT_WARPS * 32) k_slots(const int32_t* __restrict__ idx, int T,
                                                           int K, int N,
                                                           const int32_t* __restrict__ base,
                                                           int32_t* __restrict__ slot_of,
                                                           int32_t* __restrict__ perm_src) {
  grid_dep_sync();
  extern __shared__ int32_t sub[];            // [SLOT_WARPS][N] counts, then first rows
  const int lane = lane_id(), w = warp_id();
  for (int i = threadIdx.x; i < SLOT_WARPS * N; i += blockDim.x) sub[i] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * CHUNK + w * SLOT_TOKENS;
  const int t1 = min(T, t0 + SLOT_TOKENS);
  for (int i = t0 * K + lane; i < t1 * K; i += 32) {
    const int e = idx[i];
    if ((unsigned)e < (unsigned)N) atomicAdd(&sub[w * N + e], 1);
  }
  __syncthreads();
  // exclusive prefix over the warps, seeded with the chunk's first row per expert
  for (int e = threadIdx.x; e < N; e += blockDim.x) {
    int run = base[(size_t)blockIdx.x * N + e];
#pragma unroll
    for (int j = 0; j < SLOT_WARPS; ++j) {
      const int c = sub[j * N + e];
      sub[j * N + e] = run;
      run += c;
    }
  }
  __syncthreads();
  int32_t* next = sub + w * N;
  for (int t = t0; t < t1; ++t) {
    if (lane < K) {
      const int e = idx[(size_t)t * K + lane];
      if ((unsigned)e < (unsigned)N) {
        const int row = next[e];
        next[e] = row + 1;
        slot_of[(size_t)t * K + lane] = row;
        perm_src[row] = t;
      } else {
        slot_of[(size_t)t * K + lane] = -1;
      }
    }
    __syncwarp();
  }
}

// Row gather x -> x_perm (fp32 / bf16) on the bulk-copy engine: one thread
// per CTA streams its tokens (t = blockIdx.x, += gridDim.x) through a ring of
// GATHER_BUFS row buffers in shared memory: one bulk load of the token's row,
// then K bulk stores of it to the token's permuted rows (one bulk group per
// token).  GATHER_BUFS - 1 loads are in flight ahead of the stores; a buffer is
// reloaded once the stores of the token that used it have read it.  The SM
// issues a handful of instructions per row, so the copy keeps its pace when
// the SM clock drops under the power limit.
constexpr int GATHER_BUFS = 4;

__host__ __device__ inline size_t gather_smem_bytes(int row_bytes) {
  return 128 + (size_t)GATHER_BUFS * row_bytes + 128;   // barriers, then the 128-aligned rows
}

__global__ void __launch_bounds__(32) k_gather(const uint8_t* __restrict__ x, int T, int K,
                                               int row_bytes, const int32_t* __restrict__ slot_of,
                                               uint8_t* __restrict__ x_perm) {
  grid_dep_sync();
  extern __shared__ __align__(16) uint8_t gather_raw[];
  if (threadIdx.x != 0) return;
  uint64_t* bar = reinterpret_cast<uint64_t*>(gather_raw);
  uint8_t* buf = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gather_raw) + 128 + 127) &
                                            ~static_cast<uintptr_t>(127));
  for (int j = 0; j < GATHER_BUFS; ++j) mbar_init(&bar[j], 1);
  fence_barrier_init();
  const int R = T * K;
  const int first = blockIdx.x, step = gridDim.x;
  const int n_my = first < T ? (T - 1 - first) / step + 1 : 0;
  auto load = [&](int i) {
    const int j = i % GATHER_BUFS;
    mbar_arrive_expect_tx(&bar[j], (uint32_t)row_bytes);
    bulk_load_1d(buf + (size_t)j * row_bytes, x + (size_t)(first + i * step) * row_bytes,
                 (uint32_t)row_bytes, &bar[j]);
  };
  for (int i = 0; i < GATHER_BUFS - 1 && i < n_my; ++i) load(i);
  volatile int no_abort = 0;
  for (int i = 0; i < n_my; ++i) {
    const int t = first + i * step, j = i % GATHER_BUFS;
    if (!mbar_wait(&bar[j], (uint32_t)(i / GATHER_BUFS) & 1u, &no_abort)) {
      // gave up (status set): let the loads already issued land before leaving
      for (int i2 = i; i2 < i + GATHER_BUFS - 1 && i2 < n_my; ++i2)
        mbar_wait(&bar[i2 % GATHER_BUFS], (uint32_t)(i2 / GATHER_BUFS) & 1u, &no_abort);
      break;
    }
    const uint8_t* src = buf + (size_t)j * row_bytes;
    for (int k = 0; k < K; ++k) {
      const int row = slot_of[(size_t)t * K + k];
      if ((unsigned)row >= (unsigned)R) continue;  // invalid pair (already reported)
      bulk_store_1d(x_perm + (size_t)row * row_bytes, src, (uint32_t)row_bytes);
    }
    bulk_commit_group();
    if (i + GATHER_BUFS - 1 < n_my) {
      // the buffer of token i - 1 is next: its stores have read it
      bulk_wait_group_read<1>();
      load(i + GATHER_BUFS - 1);
    }
  }
  bulk_wait_group_all();
}

// bf16 row -> E4M3 codes per 1x128 tile, written to the token's K permuted rows
// and to row R + t (the shared experts' input), with the fp32 tile scales.
// Scale rule: amax = max|v|, scale = amax / 448, code = E4M3(v * (448 / amax))
// rounded to nearest even with saturation; amax = 0 gives scale 0, codes 0.
// One warp quantises the 1x128 tile g of a bf16 row: lane l takes elements
// 4l .. 4l+3 and returns their E4M3 codes packed little-endian, and every lane
// the tile's fp32 scale (amax / 448; 0 for an all-zero tile).
__device__ __forceinline__ void quant_tile_1x128(const __nv_bfloat16* __restrict__ xr, int g,
                                                 int lane, uint32_t& code, float& scale) {
  const uint2 raw = *reinterpret_cast<const uint2*>(xr + g * 128 + lane * 4);
  const __nv_bfloat162 p0 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
  const __nv_bfloat162 p1 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
  const float v0 = __low2float(p0), v1 = __high2float(p0), v2 = __low2float(p1),
              v3 = __high2float(p1);
  const float amax = warp_max(fmaxf(fmaxf(fabsf(v0), fabsf(v1)), fmaxf(fabsf(v2), fabsf(v3))));
  scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 0.f;
  const float inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 0.f;
  code = (uint32_t)f32_to_e4m3(__fmul_rn(v0, inv)) |
         ((uint32_t)f32_to_e4m3(__fmul_rn(v1, inv)) << 8) |
         ((uint32_t)f32_to_e4m3(__fmul_rn(v2, inv)) << 16) |
         ((uint32_t)f32_to_e4m3(__fmul_rn(v3, inv)) << 24);
}

__global__ void __launch_bounds__(256) k_gather_quant(const __nv_bfloat16* __restrict__ x, int T,
                                                      int K, int d, int R,
                                                      const int32_t* __restrict__ slot_of,
                                                      uint8_t* __restrict__ xq,
                                                      float* __restrict__ xs) {
  grid_dep_sync();
  const int t = blockIdx.x * 8 + warp_id();
  if (t >= T) return;
  const int lane = lane_id();
  const int ng = d / 128;
  int my_slot = lane < K ? slot_of[(size_t)t * K + lane] : 0;
  const __nv_bfloat16* xr = x + (size_t)t * d;
  for (int g = 0; g < ng; ++g) {
    uint32_t code;
    float scale;
    quant_tile_1x128(xr, g, lane, code, scale);
    for (int k = 0; k <= K; ++k) {
      const int row = k < K ? __shfl_sync(0xffffffffu, my_slot, k) : R + t;
      if (k < K && (unsigned)row >= (unsigned)R) continue;  // invalid pair (already reported)
      *reinterpret_cast<uint32_t*>(xq + (size_t)row * d + g * 128 + lane * 4) = code;
      if (lane == 0) xs[(size_t)row * ng + g] = scale;
    }
  }
}

// Group table for the grouped GEMMs (block 0) and the permuted-row -> pair map
// (all blocks).  Groups: shared experts 0..Ks-1 then routed experts 0..N-1.
__global__ void __launch_bounds__(1024) k_prep_groups(const int32_t* __restrict__ offsets, int T,
                                                      int K, int Ks, int N, int fp8,
                                                      int32_t* __restrict__ gtab,
                                                      const int32_t* __restrict__ slot_of,
                                                      int32_t* __restrict__ pair_of) {
  grid_dep_sync();
  const int R = T * K;
  if (blockIdx.x > 0) {
    for (int i = (blockIdx.x - 1) * blockDim.x + threadIdx.x; i < R;
         i += (gridDim.x - 1) * blockDim.x) {
      const int row = slot_of[i];
      if ((unsigned)row < (unsigned)R) pair_of[row] = i;
      else set_status(MOE_ERR_DEVICE_CHECK);
    }
    return;
  }
  __shared__ int32_t warp_tot[32];
  const int n = Ks + N;
  int32_t* prefix = gtab;
  int32_t* rows = gtab + n + 1;
  int32_t* a_row = rows + n;
  int32_t* a_map = a_row + n;
  int32_t* expert = a_map + n;
  int32_t* c_row = expert + n;
  int32_t* aux = c_row + n;
  // n <= blockDim.x (checked on the host): one thread per group.
  const int g = threadIdx.x;
  int mtiles = 0;
  if (g < n) {
    int rws, ar, am, cr, ax;
    if (g < Ks) {
      rws = T;
      am = fp8 ? 1 : 0;
      ar = fp8 ? R : 0;
      cr = R + g * T;
      ax = g;
    } else {
      const int j = g - Ks;
      const int o0 = offsets[j], o1 = offsets[j + 1];
      rws = o1 - o0;
      if (rws < 0 || o0 < 0 || o1 > R) { set_status(MOE_ERR_DEVICE_CHECK); rws = 0; }
      am = 1;
      ar = o0;
      cr = o0;
      ax = -1;
    }
    rows[g] = rws;
    a_row[g] = ar;
    a_map[g] = am;
    expert[g] = g;
    c_row[g] = cr;
    aux[g] = ax;
    mtiles = (rws + gemm::BM - 1) / gemm::BM;
  }
  int incl = mtiles;
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
  const int excl = incl - mtiles + warp_tot[warp_id()];
  if (g < n) prefix[g] = excl;
  if (g == n - 1) prefix[n] = excl + mtiles;
}

// h[t] = x_res[t] + sum_{s<Ks} y[t, K+s] + sum_{k<K} y[t, k], fp32, in that order.
// Each thread owns 8 consecutive elements (bf16) or 4 (fp32) of one token.
template <bool BF16>
__global__ void __launch_bounds__(256) k_combine(const void* __restrict__ x_res,
                                                 const void* __restrict__ y, void* __restrict__ h,
                                                 int T, int d, int K, int Ks) {
  grid_dep_sync();
  constexpr int VEC = BF16 ? 8 : 4;
  const int per_tok = d / VEC;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)T * per_tok) return;
  const int t = (int)(gid / per_tok);
  const int c = (int)(gid - (long long)t * per_tok) * VEC;
  const int S = K + Ks;
  float acc[VEC];
  auto load = [&](const void* base, long long elem_off, float (&v)[VEC]) {
    if (BF16) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(
          reinterpret_cast<const __nv_bfloat16*>(base) + elem_off));
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int i = 0; i < VEC / 2; ++i) {
        v[2 * i] = __low2float(p[i]);
        v[2 * i + 1] = __high2float(p[i]);
      }
    } else {
      const float4 raw = __ldg(reinterpret_cast<const float4*>(
          reinterpret_cast<const float*>(base) + elem_off));
      v[0] = raw.x; v[1] = raw.y; v[2] = raw.z; v[3] = raw.w;
    }
  };
  load(x_res, (long long)t * d + c, acc);
  const long long ybase = (long long)t * S * d + c;
  for (int s = 0; s < Ks; ++s) {
    float v[VEC];
    load(y, ybase + (long long)(K + s) * d, v);
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] += v[i];
  }
  for (int k = 0; k < K; ++k) {
    float v[VEC];
    load(y, ybase + (long long)k * d, v);
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] += v[i];
  }
  if (BF16) {
    uint4 out;
    uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = gemm::pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(h) + (long long)t * d + c) = out;
  } else {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(h) + (long long)t * d + c) =
        make_float4(acc[0], acc[1], acc[2], acc[3]);
  }
}

// Destinations of a dispatch straight into the ranks' receive buffers: the
// send-order rows [start[q], start[q+1]) go to rows base[q] + (row - start[q])
// of rank q's buffers x[q] (rows) and w[q] (gate weights).  The addresses may
// be other GPUs' memory (CUDA IPC mappings); the kernel only stores to them.
constexpr int MAX_PEERS = 16;
struct PeerDest {
  uint8_t* x[MAX_PEERS];
  float* w[MAX_PEERS];
  float* s[MAX_PEERS];     // E4M3 rows: the 1x128 tile scales of the rows
  int start[MAX_PEERS + 1];
  int base[MAX_PEERS];
  int n;
};

// Dispatch gather (expert parallelism): the send-order row row_of[t*K + k]
// receives x[t] and topk_w[t*K + k].  Local (PEER = false): row r of x_rows /
// w_rows (and of the tile scales s_rows).  PEER: the row's rank and place from
// the PeerDest table.  FP8: x is bf16 and each 1x128 tile is quantised to
// E4M3 once (codes and fp32 scale, as the layer's gather does) before its K
// copies are stored.  One warp per token reads its row once and writes it to
// its K rows.
template <bool PEER, bool FP8>
__global__ void __launch_bounds__(256) k_dispatch_rows(const uint8_t* __restrict__ x, int T,
                                                       int K, int row_bytes,
                                                       const float* __restrict__ topk_w,
                                                       const int32_t* __restrict__ row_of,
                                                       int n_rows, uint8_t* __restrict__ x_rows,
                                                       float* __restrict__ w_rows,
                                                       float* __restrict__ s_rows,
                                                       const PeerDest P) {
  grid_dep_sync();
  const int t = blockIdx.x * 8 + warp_id();
  if (t >= T) return;
  const int lane = lane_id();
  const int ng = row_bytes / 128;      // FP8: row_bytes = d
  uint8_t* my_dst = nullptr;
  float* my_sdst = nullptr;
  if (lane < K) {
    const int row = row_of[(size_t)t * K + lane];
    if ((unsigned)row >= (unsigned)n_rows) {
      set_status(MOE_ERR_DEVICE_CHECK);
    } else if (!PEER) {
      my_dst = x_rows + (size_t)row * row_bytes;
      if (FP8) my_sdst = s_rows + (size_t)row * ng;
      if (w_rows) w_rows[row] = topk_w[(size_t)t * K + lane];
    } else {
      int q = 0;
      while (q + 1 < P.n && row >= P.start[q + 1]) ++q;
      const size_t r = (size_t)P.base[q] + (size_t)(row - P.start[q]);
      my_dst = P.x[q] + r * row_bytes;
      if (FP8) my_sdst = P.s[q] + r * ng;
      if (P.w[q]) P.w[q][r] = topk_w[(size_t)t * K + lane];
    }
  }
  if (FP8) {
    const __nv_bfloat16* xr = reinterpret_cast<const __nv_bfloat16*>(x) + (size_t)t * row_bytes;
    for (int g = 0; g < ng; ++g) {
      uint32_t code;
      float scale;
      quant_tile_1x128(xr, g, lane, code, scale);
      for (int k = 0; k < K; ++k) {
        uint8_t* dst = reinterpret_cast<uint8_t*>(
            __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(my_dst), k));
        float* sdst = reinterpret_cast<float*>(
            __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(my_sdst), k));
        if (dst) {
          *reinterpret_cast<uint32_t*>(dst + g * 128 + lane * 4) = code;
          if (lane == 0) sdst[g] = scale;
        }
      }
    }
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * row_bytes);
  const int nvec = row_bytes / 16;
  for (int c0 = 0; c0 < nvec; c0 += 32) {
    const int c = c0 + lane;
    const bool in = c < nvec;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (in) v = __ldg(src + c);
    for (int k = 0; k < K; ++k) {
      uint8_t* dst = reinterpret_cast<uint8_t*>(
          __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(my_dst), k));
      if (in && dst) reinterpret_cast<uint4*>(dst)[c] = v;
    }
  }
}

// 1x128 E4M3 quantisation of n bf16 rows of d elements (one warp a row):
// codes [n, d], scales [n, d / 128].
__global__ void __launch_bounds__(256) k_quant_rows(const __nv_bfloat16* __restrict__ x, int n,
                                                    int d, uint8_t* __restrict__ codes,
                                                    float* __restrict__ scales) {
  grid_dep_sync();
  const int t = blockIdx.x * 8 + warp_id();
  if (t >= n) return;
  const int lane = lane_id(), ng = d / 128;
  const __nv_bfloat16* xr = x + (size_t)t * d;
  for (int g = 0; g < ng; ++g) {
    uint32_t code;
    float scale;
    quant_tile_1x128(xr, g, lane, code, scale);
    *reinterpret_cast<uint32_t*>(codes + (size_t)t * d + g * 128 + lane * 4) = code;
    if (lane == 0) scales[(size_t)t * ng + g] = scale;
  }
}

// Group table of a caller-given list of row groups (expert parallelism): group
// i reads rows [row0, row0 + rows) of x_rows with expert `expert` and writes
// rows [out0, out0 + rows) of H and of the output.  One block; n <= 1024.
__global__ void __launch_bounds__(1024) k_prep_user_groups(const int32_t* __restrict__ groups,
                                                           int n, int n_experts, int n_in,
                                                           int n_out, int32_t* __restrict__ gtab) {
  grid_dep_sync();
  __shared__ int32_t warp_tot[32];
  int32_t* prefix = gtab;
  int32_t* rows = gtab + n + 1;
  int32_t* a_row = rows + n;
  int32_t* a_map = a_row + n;
  int32_t* expert = a_map + n;
  int32_t* c_row = expert + n;
  int32_t* aux = c_row + n;
  const int g = threadIdx.x;
  int mtiles = 0;
  if (g < n) {
    const int r0 = groups[4 * g], rw = groups[4 * g + 1], ex = groups[4 * g + 2],
              o0 = groups[4 * g + 3];
    const bool ok = rw >= 0 && r0 >= 0 && o0 >= 0 && (long long)r0 + rw <= n_in &&
                    (long long)o0 + rw <= n_out && ex >= 0 && ex < n_experts;
    if (!ok) set_status(MOE_ERR_DEVICE_CHECK);
    rows[g] = ok ? rw : 0;
    a_row[g] = ok ? r0 : 0;
    a_map[g] = 1;
    expert[g] = ok ? ex : 0;
    c_row[g] = ok ? o0 : 0;
    aux[g] = -1;
    mtiles = ok ? (rw + gemm::BM - 1) / gemm::BM : 0;
  }
  int incl = mtiles;
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
  const int excl = incl - mtiles + warp_tot[warp_id()];
  if (g < n) prefix[g] = excl;
  if (g == n - 1) prefix[n] = excl + mtiles;
}

// h[t] = x_res[t] + sum_{s<Ks} y_shared[s*T + t] + sum_{k<K} y_rows[row_of[t*K + k]],
// fp32, in that order (the order of k_combine, so the two agree bit for bit
// when the rows hold the same values).  A row index outside [0, n_rows) is
// reported and skipped.
template <bool BF16>
__global__ void __launch_bounds__(256) k_combine_rows(const void* __restrict__ x_res,
                                                      const void* __restrict__ y_shared,
                                                      const void* __restrict__ y_rows,
                                                      const int32_t* __restrict__ row_of,
                                                      int n_rows, void* __restrict__ h, int T,
                                                      int d, int K, int Ks) {
  grid_dep_sync();
  constexpr int VEC = BF16 ? 8 : 4;
  const int per_tok = d / VEC;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)T * per_tok) return;
  const int t = (int)(gid / per_tok);
  const int c = (int)(gid - (long long)t * per_tok) * VEC;
  float acc[VEC];
  auto load = [&](const void* base, long long elem_off, float (&v)[VEC]) {
    if (BF16) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(
          reinterpret_cast<const __nv_bfloat16*>(base) + elem_off));
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int i = 0; i < VEC / 2; ++i) {
        v[2 * i] = __low2float(p[i]);
        v[2 * i + 1] = __high2float(p[i]);
      }
    } else {
      const float4 raw = __ldg(reinterpret_cast<const float4*>(
          reinterpret_cast<const float*>(base) + elem_off));
      v[0] = raw.x; v[1] = raw.y; v[2] = raw.z; v[3] = raw.w;
    }
  };
  load(x_res, (long long)t * d + c, acc);
  for (int s = 0; s < Ks; ++s) {
    float v[VEC];
    load(y_shared, ((long long)s * T + t) * d + c, v);
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] += v[i];
  }
  for (int k = 0; k < K; ++k) {
    const int r = row_of[(size_t)t * K + k];
    if ((unsigned)r >= (unsigned)n_rows) {
      if (c == 0) set_status(MOE_ERR_DEVICE_CHECK);
      continue;
    }
    float v[VEC];
    load(y_rows, (long long)r * d + c, v);
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] += v[i];
  }
  if (BF16) {
    uint4 out;
    uint32_t* o = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = gemm::pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
    *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(h) + (long long)t * d + c) = out;
  } else {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(h) + (long long)t * d + c) =
        make_float4(acc[0], acc[1], acc[2], acc[3]);
  }
}

// 128x128 block quantisation of bf16 weights to E4M3 (same rule as the
// activation tiles).  One block of 256 threads per weight block.
// TRANSPOSE: the codes and scales of the transposed matrix, [cols, rows] and
// [cols / 128, rows / 128] (a block's amax does not depend on its
// orientation, so these are the transposed matrix's own codes and scales).
template <bool TRANSPOSE>
__global__ void __launch_bounds__(256) k_quant_w(const __nv_bfloat16* __restrict__ w, int rows,
                                                 int cols, uint8_t* __restrict__ q,
                                                 float* __restrict__ scale) {
  __shared__ float red[8];
  __shared__ __align__(16) uint8_t tile[TRANSPOSE ? 128 : 1][TRANSPOSE ? 128 + 16 : 1];
  const int bc = cols / 128, br = rows / 128;
  const int b = blockIdx.x;  // over batch * br * bc
  const int mat = b / (br * bc), rem = b - mat * br * bc;
  const int bi = rem / bc, bj = rem - bi * bc;
  const __nv_bfloat16* src = w + (size_t)mat * rows * cols + (size_t)bi * 128 * cols + bj * 128;
  uint8_t* dst = q + (size_t)mat * rows * cols + (size_t)bi * 128 * cols + bj * 128;
  // each thread: rows r = tid/2 (128 rows, 2 threads per row), 64 columns
  const int r = threadIdx.x >> 1, half = threadIdx.x & 1;
  const __nv_bfloat16* rp = src + (size_t)r * cols + half * 64;
  float v[64];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 raw = *reinterpret_cast<const uint4*>(rp + i * 8);
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[i * 8 + 2 * j] = __low2float(p[j]);
      v[i * 8 + 2 * j + 1] = __high2float(p[j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fabsf(v[i]));
  amax = warp_max(amax);
  if (lane_id() == 0) red[warp_id()] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float sc = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 0.f;
  const float inv = amax > 0.f ? __fdiv_rn(448.0f, amax) : 0.f;
  uint8_t* dp = TRANSPOSE ? &tile[r][half * 64] : dst + (size_t)r * cols + half * 64;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t wds[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int o = i * 16 + j * 4;
      wds[j] = (uint32_t)f32_to_e4m3(__fmul_rn(v[o], inv)) |
               ((uint32_t)f32_to_e4m3(__fmul_rn(v[o + 1], inv)) << 8) |
               ((uint32_t)f32_to_e4m3(__fmul_rn(v[o + 2], inv)) << 16) |
               ((uint32_t)f32_to_e4m3(__fmul_rn(v[o + 3], inv)) << 24);
    }
    *reinterpret_cast<uint4*>(dp + i * 16) = make_uint4(wds[0], wds[1], wds[2], wds[3]);
  }
  if (TRANSPOSE) {
    // block (bi, bj) of the codes becomes block (bj, bi) of the transpose:
    // thread (c, half) writes 64 bytes of output row c, read down a column
    __syncthreads();
    const int c = threadIdx.x >> 1;
    uint8_t* tp = q + (size_t)mat * rows * cols + ((size_t)bj * 128 + c) * rows + bi * 128 +
                  half * 64;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t wds[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r0 = half * 64 + i * 16 + j * 4;
        wds[j] = (uint32_t)tile[r0][c] | ((uint32_t)tile[r0 + 1][c] << 8) |
                 ((uint32_t)tile[r0 + 2][c] << 16) | ((uint32_t)tile[r0 + 3][c] << 24);
      }
      *reinterpret_cast<uint4*>(tp + i * 16) = make_uint4(wds[0], wds[1], wds[2], wds[3]);
    }
    if (threadIdx.x == 0) scale[(size_t)mat * br * bc + bj * br + bi] = sc;
  } else {
    if (threadIdx.x == 0) scale[(size_t)mat * br * bc + bi * bc + bj] = sc;
  }
}

}  // namespace perm
}  // namespace moe
