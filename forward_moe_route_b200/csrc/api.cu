// C ABI of the DeepSeekMoE layer forward (declared in include/moe.h): argument
// validation, workspace layout, tensor-map encoding and kernel launches.
//
// All kernels live in this one translation unit, so the per-device status
// word is a single __device__ variable that every kernel names directly.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "gemm.cuh"
#include "gemm_fp8.cuh"
#include "gemm_t.cuh"
#include "gemm_gu.cuh"
#include "permute.cuh"
#include "route.cuh"
#include "bwd.cuh"
#include "bwd8.cuh"
#include "gemm_bwd.cuh"

using namespace moe;

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kAlign = 256;
constexpr int kMaxShared = 64;     // shared experts accepted
constexpr int kMaxRouted = 512;
constexpr int kMaxSmem = 232448;   // dynamic shared memory per block on sm_100

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Dims {
  int64_t T, d, Ks, N, K, I, E, R;
  int act, w;
  bool fp8, f32;
  size_t x_esz;   // bytes per element of x, w_router and x_residual
  size_t op_esz;  // bytes per element of the GEMM operands x_perm and H
  size_t y_esz;   // bytes per element of y_slots and h
  int n_chunks;
};

moe_status fill_dims(const moe_layer_desc* desc, Dims* D) {
  if (!desc) return MOE_ERR_INVALID_ARG;
  const moe_layer_desc& s = *desc;
  if (s.T < 0 || s.d < 1 || s.n_shared < 0 || s.n_shared > kMaxShared || s.n_routed < 1 ||
      s.n_routed > kMaxRouted || s.top_k < 1 || s.top_k > route::MAXK || s.top_k > s.n_routed ||
      s.inter < 16 || s.d > 65536 || s.inter > 65536)
    return MOE_ERR_INVALID_ARG;
  if (s.gate != MOE_GATE_SOFTMAX && s.gate != MOE_GATE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (s.renorm != 0 && s.renorm != 1) return MOE_ERR_INVALID_ARG;
  if (!std::isfinite(s.route_scale) || !(s.route_scale > 0.f)) return MOE_ERR_INVALID_ARG;
  if (s.n_group < 1 || s.n_group > 32 || s.topk_group < 1 || s.topk_group > s.n_group ||
      s.n_routed % s.n_group != 0)
    return MOE_ERR_INVALID_ARG;
  if (s.n_group > 1 && (s.n_routed / s.n_group < 2 ||
                        (int64_t)s.topk_group * (s.n_routed / s.n_group) < s.top_k))
    return MOE_ERR_INVALID_ARG;
  int align;
  if (s.act_dtype == MOE_DT_F32 && s.w_dtype == MOE_DT_F32) {
    D->x_esz = 4; D->op_esz = 4; D->y_esz = 4; align = 32; D->fp8 = false; D->f32 = true;
  } else if (s.act_dtype == MOE_DT_BF16 && s.w_dtype == MOE_DT_BF16) {
    D->x_esz = 2; D->op_esz = 2; D->y_esz = 2; align = 64; D->fp8 = false; D->f32 = false;
  } else if (s.act_dtype == MOE_DT_BF16 && s.w_dtype == MOE_DT_E4M3) {
    D->x_esz = 2; D->op_esz = 1; D->y_esz = 2; align = 128; D->fp8 = true; D->f32 = false;
  } else {
    return MOE_ERR_INVALID_ARG;
  }
  if (s.d % align || s.inter % align) return MOE_ERR_INVALID_ARG;
  D->T = s.T; D->d = s.d; D->Ks = s.n_shared; D->N = s.n_routed; D->K = s.top_k; D->I = s.inter;
  D->E = D->Ks + D->N;
  D->R = D->T * D->K;
  D->act = s.act_dtype; D->w = s.w_dtype;
  if (D->R + D->Ks * D->T + D->T >= ((int64_t)1 << 31)) return MOE_ERR_INVALID_ARG;
  D->n_chunks = (int)((D->T + perm::CHUNK - 1) / perm::CHUNK);
  return MOE_OK;
}

struct Layout {
  size_t logits, topk_idx, topk_w, counts, hist, offsets, perm_src, slot_of, pair_of, gtab;
  size_t x_perm, x_perm_scale, hbuf, hscale, y_slots, total;
};

Layout layout(const Dims& D) {
  Layout L;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, kAlign); return at; };
  L.logits = take(D.f32 ? 0 : (size_t)D.T * D.N * 4);
  L.topk_idx = take((size_t)D.R * 4);
  L.topk_w = take((size_t)D.R * 4);
  L.counts = take((size_t)D.N * 4);
  L.hist = take((size_t)(D.n_chunks > 0 ? D.n_chunks : 1) * D.N * 4);
  L.offsets = take((size_t)(D.N + 1) * 4);
  L.perm_src = take((size_t)D.R * 4);
  L.slot_of = take((size_t)D.R * 4);
  L.pair_of = take((size_t)D.R * 4);
  L.gtab = take((size_t)gemm::group_tab_ints((int)D.E) * 4);
  const size_t xrows = (size_t)D.R + (D.fp8 ? (size_t)D.T : 0);
  L.x_perm = take(xrows * D.d * D.op_esz);
  L.x_perm_scale = take(D.fp8 ? xrows * (D.d / 128) * 4 : 0);
  const size_t hrows = (size_t)D.R + (size_t)D.Ks * D.T;
  L.hbuf = take(hrows * D.I * D.op_esz);
  L.hscale = take(D.fp8 ? hrows * (D.I / 128) * 4 : 0);
  L.y_slots = take((size_t)D.T * (D.K + D.Ks) * D.d * D.y_esz);
  L.total = o;
  return L;
}

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// ----------------------------------------------------------------------------- device setup
struct DeviceInfo {
  int sms = 0;
  bool attrs_done = false;
  // co-resident 2-CTA clusters of the pair GEMMs (0: gate/up, 1: down,
  // 2: backward weight gradients, 3: backward activation GEMMs), and the
  // dynamic shared memory each count was taken for
  size_t pair_smem[4] = {0, 0, 0, 0};
  int pair_clusters[4] = {0, 0, 0, 0};
};
std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;


template <int KIND>
cudaError_t set_down_attr() {
  cudaError_t e = cudaFuncSetAttribute(gemmt::k_down_gemm<KIND>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemmgu::k_gate_up_gemm<KIND>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  return e;
}

// Text of the last CUDA failure on this host thread (moe_last_error_message).
thread_local char t_errmsg[256] = "";

moe_status cuda_fail(cudaError_t e, const char* where) {
  snprintf(t_errmsg, sizeof(t_errmsg), "%s: %s (%s)", where, cudaGetErrorName(e),
           cudaGetErrorString(e));
  return MOE_ERR_CUDA;
}

moe_status device_setup(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.attrs_done) {
    if (cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess) e = set_down_attr<0>();
    if (e == cudaSuccess) e = set_down_attr<1>();
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(perm::k_gather, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kMaxSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm8::k_gemm_promoted<0, gemm8::EPI_F32_STORE>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm8::k_gemm_promoted<2, gemm8::EPI_SWIGLU_Q>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm8::k_gemm_promoted<2, gemm8::EPI_SCATTER>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm8::k_gemm_promoted<2, gemm8::EPI_BF16_OUT>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm8::k_gemm_promoted<2, gemm8::EPI_SWIGLU_BWD>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm8::k_gemm_promoted<2, gemm8::EPI_BF16_OUT, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute (dynamic shared memory)");
    // the promoted GEMMs re-split their registers with setmaxnreg; the split
    // adds up only if a thread starts with exactly LAUNCH_REGS registers
    {
      cudaFuncAttributes fa[6];
      if (cudaFuncGetAttributes(&fa[0], gemm8::k_gemm_promoted<0, gemm8::EPI_F32_STORE>) !=
              cudaSuccess ||
          cudaFuncGetAttributes(&fa[1], gemm8::k_gemm_promoted<2, gemm8::EPI_SWIGLU_Q>) !=
              cudaSuccess ||
          cudaFuncGetAttributes(&fa[2], gemm8::k_gemm_promoted<2, gemm8::EPI_SCATTER>) !=
              cudaSuccess ||
          cudaFuncGetAttributes(&fa[3], gemm8::k_gemm_promoted<2, gemm8::EPI_BF16_OUT>) !=
              cudaSuccess ||
          cudaFuncGetAttributes(&fa[4], gemm8::k_gemm_promoted<2, gemm8::EPI_SWIGLU_BWD>) !=
              cudaSuccess ||
          cudaFuncGetAttributes(&fa[5], gemm8::k_gemm_promoted<2, gemm8::EPI_BF16_OUT, true>) !=
              cudaSuccess)
        return MOE_ERR_CUDA;
      for (const auto& f : fa)
        if (f.numRegs != gemm8::LAUNCH_REGS) {
          snprintf(t_errmsg, sizeof(t_errmsg),
                   "promoted GEMM compiled with %d registers a thread, expected %d", f.numRegs,
                   gemm8::LAUNCH_REGS);
          return MOE_ERR_UNSUPPORTED;
        }
    }
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return MOE_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    di.attrs_done = true;
  }
  *sms = di.sms;
  return MOE_OK;
}


inline moe_status launched(const char* where) {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, where);
}

// Launch one kernel of the layer's chain with programmatic stream
// serialisation: its launch may overlap the end of the previous kernel on the
// stream; the kernel itself waits for that kernel's results (grid_dep_sync).
template <typename... KArgs, typename... Args>
moe_status launch_chain(const char* what, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                        size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, what);
}

// 2-D K-major tensor map with 128-byte swizzle: rows of `inner` elements,
// box = (128 bytes of K) x box_rows.
moe_status make_tmap(CUtensorMap* m, const void* base, size_t esz, uint64_t inner, uint64_t rows,
                     uint32_t box_rows) {
  CUtensorMapDataType dt = esz == 4   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                           : esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                      : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  cuuint64_t dims[2] = {inner, rows > 0 ? rows : 1};
  cuuint64_t strides[1] = {inner * esz};
  cuuint32_t box[2] = {(cuuint32_t)(gemm::KB / esz), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(t_errmsg, sizeof(t_errmsg), "cuTensorMapEncodeTiled: CUresult %d (rows %llu, "
             "inner %llu, box rows %u)", (int)r, (unsigned long long)rows,
             (unsigned long long)inner, box_rows);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}



// Stage-timing events of the calling host thread (moe_trace_events).
thread_local cudaEvent_t* t_events = nullptr;
inline moe_status trace(int i, cudaStream_t st) {
  if (!t_events) return MOE_OK;
  const cudaError_t e = cudaEventRecord(t_events[i], st);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "cudaEventRecord (stage trace)");
}






route::Params route_params(const moe_layer_desc& s) {
  route::Params p;
  p.T = s.T; p.N = s.n_routed; p.K = s.top_k; p.gate = s.gate; p.renorm = s.renorm;
  p.n_group = s.n_group; p.topk_group = s.topk_group; p.scale = s.route_scale;
  return p;
}

template <int VPL>
moe_status launch_topk(const float* logits, const float* bias, const route::Params& p,
                       int32_t* idx, float* w, cudaStream_t st) {
  return launch_chain("k_topk", route::k_topk<VPL>, dim3((p.T + 7) / 8), dim3(256), 0, st,
                      logits, bias, p, idx, w);
}
template <int VPL>
moe_status launch_route_f32(const float* x, const float* wr, int d, const float* bias,
                            const route::Params& p, int32_t* idx, float* w, cudaStream_t st) {
  return launch_chain("k_route_f32", route::k_route_f32<VPL>, dim3((p.T + 7) / 8), dim3(256), 0,
                      st, x, wr, d, bias, p, idx, w);
}

// ----------------------------------------------------------------------------- stages
// bf16 router GEMM on tensor cores: logits [T, N] fp32.  Each 64-element K
// block is a separate tensor-core product added into fp32 registers with
// round-to-nearest, so the logits keep fp32 accuracy over the whole of d (the
// selection is decided on them).  Its prologue zeroes `zero_counts` (if any).
moe_status launch_router(const Dims& D, const void* x, const void* w_router, float* logits,
                         int32_t* zero_counts, int sms, cudaStream_t st) {
  const int N = (int)D.N;
  CUtensorMap ta, tb;
  moe_status rc = make_tmap(&ta, x, 2, D.d, D.T, gemm8::BM);
  if (rc == MOE_OK) rc = make_tmap(&tb, w_router, 2, D.d, D.N, gemm8::BN);
  if (rc != MOE_OK) return rc;
  gemm8::Args a;
  memset(&a, 0, sizeof(a));
  a.gt.base = nullptr;
  a.gt.n = 1;
  a.gt.single_rows = (int)D.T;
  a.n_tiles_n = (N + gemm8::BN - 1) / gemm8::BN;
  a.num_kb = (int)(D.d * 2 / gemm8::KB);
  a.kb_elems = gemm8::KB / 2;
  a.b_rows_per_expert = 0;
  a.idesc = umma_idesc(1, gemm8::BM, gemm8::BN);
  a.out = logits;
  a.out_ld = N;
  a.out_cols = N;
  a.zero_ptr = zero_counts;
  a.zero_n = zero_counts ? N : 0;
  int stages = 0;
  for (int s = 6; s >= 2 && !stages; --s)
    if (gemm8::smem_bytes(s, 1) <= (size_t)kMaxSmem) stages = s;
  a.stages = stages;
  const int tiles = (int)((D.T + 127) / 128) * a.n_tiles_n;
  return launch_chain("router GEMM", gemm8::k_gemm_promoted<0, gemm8::EPI_F32_STORE>,
                      dim3(tiles < sms ? tiles : sms), dim3(gemm8::NUM_THREADS),
                      gemm8::smem_bytes(stages, 1), st, ta, tb, a);
}

// The per-chunk histogram scan, with 16-byte loads along the rows when N % 4 == 0.
moe_status launch_scan(cudaStream_t st, int32_t* hist, int n_chunks, int N,
                       const int32_t* counts, int32_t* counts_out, int32_t* offsets) {
  if (N % 4 == 0)
    return launch_chain("k_scan", perm::k_scan<4>, dim3(1), dim3(1024), 0, st, hist, n_chunks, N,
                        counts, counts_out, offsets);
  return launch_chain("k_scan", perm::k_scan<1>, dim3(1), dim3(1024), 0, st, hist, n_chunks, N,
                      counts, counts_out, offsets);
}

// Selection and gate weights.  With counts != nullptr the tokens per expert
// are counted too: the per-chunk histogram and its totals (k_hist, k_scan),
// which the layer forward instead takes from its permutation step.
moe_status do_route(const moe_layer_desc& s, const Dims& D, const Layout& L, const void* x,
                    const void* w_router, const float* bias, int32_t* topk_idx, float* topk_w,
                    int32_t* counts, uint8_t* ws, int sms, cudaStream_t st) {
  const route::Params p = route_params(s);
  const int N = (int)D.N;
  if (D.T == 0)
    return counts ? launch_chain("k_zero_i32", route::k_zero_i32, dim3(1), dim3(256), 0, st,
                                 counts, N)
                  : MOE_OK;
  moe_status rc;
  if (D.f32) {
    const float* xf = static_cast<const float*>(x);
    const float* wf = static_cast<const float*>(w_router);
    const int dd = (int)D.d;
    if (N <= 32) rc = launch_route_f32<1>(xf, wf, dd, bias, p, topk_idx, topk_w, st);
    else if (N <= 64) rc = launch_route_f32<2>(xf, wf, dd, bias, p, topk_idx, topk_w, st);
    else if (N <= 128) rc = launch_route_f32<4>(xf, wf, dd, bias, p, topk_idx, topk_w, st);
    else if (N <= 256) rc = launch_route_f32<8>(xf, wf, dd, bias, p, topk_idx, topk_w, st);
    else rc = launch_route_f32<16>(xf, wf, dd, bias, p, topk_idx, topk_w, st);
  } else {
    float* logits = reinterpret_cast<float*>(ws + L.logits);
    rc = launch_router(D, x, w_router, logits, nullptr, sms, st);
    if (rc != MOE_OK) return rc;
    if (N <= 32) rc = launch_topk<1>(logits, bias, p, topk_idx, topk_w, st);
    else if (N <= 64) rc = launch_topk<2>(logits, bias, p, topk_idx, topk_w, st);
    else if (N <= 128) rc = launch_topk<4>(logits, bias, p, topk_idx, topk_w, st);
    else if (N <= 256) rc = launch_topk<8>(logits, bias, p, topk_idx, topk_w, st);
    else rc = launch_topk<16>(logits, bias, p, topk_idx, topk_w, st);
  }
  if (rc != MOE_OK || !counts) return rc;
  int32_t* hist = reinterpret_cast<int32_t*>(ws + L.hist);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  const int T = (int)D.T, K = (int)D.K;
  rc = launch_chain("k_hist", perm::k_hist, dim3(D.n_chunks), dim3(256), N * 4, st,
                    static_cast<const int32_t*>(topk_idx), T, K, N, hist);
  if (rc == MOE_OK)
    rc = launch_scan(st, hist, (int)D.n_chunks,
                      N, static_cast<const int32_t*>(nullptr), counts, offsets);
  return rc;
}

// hist: the per-chunk histogram scratch, ceil(T/128) x N int32 (the
// workspace's, or the fixed array of moe_permute_noalloc).
// counts: checked against the histogram's totals when given; counts_out:
// receives them when given (the layer forward's routing does not count).
moe_status do_permute(const Dims& D, int32_t* hist, const void* x, const int32_t* topk_idx,
                      const int32_t* counts, int32_t* offsets, int32_t* perm_src,
                      int32_t* slot_of, void* x_perm, float* x_perm_scale, cudaStream_t st,
                      int32_t* counts_out = nullptr) {
  const int T = (int)D.T, K = (int)D.K, N = (int)D.N;
  if (T == 0) {
    if (counts_out) {
      const moe_status rc0 = launch_chain("k_zero_i32", route::k_zero_i32, dim3(1), dim3(256), 0,
                                          st, counts_out, N);
      if (rc0 != MOE_OK) return rc0;
    }
    return launch_chain("k_zero_i32", route::k_zero_i32, dim3(1), dim3(256), 0, st, offsets,
                        N + 1);
  }
  moe_status rc = launch_chain("k_hist", perm::k_hist, dim3(D.n_chunks), dim3(256), N * 4, st,
                               topk_idx, T, K, N, hist);
  if (rc == MOE_OK)
    rc = launch_scan(st, hist, (int)D.n_chunks,
                      N, counts, counts_out, offsets);
  if (rc == MOE_OK)
    rc = launch_chain("k_slots", perm::k_slots, dim3(D.n_chunks), dim3(perm::SLOT_WARPS * 32),
                      perm::SLOT_WARPS * N * 4, st, topk_idx, T, K, N,
                      static_cast<const int32_t*>(hist), slot_of, perm_src);
  if (rc != MOE_OK) return rc;
  if (!x_perm) return MOE_OK;   // maps only (moe_permute with x_perm = NULL)
  if (D.fp8)
    return launch_chain("k_gather_quant", perm::k_gather_quant, dim3((T + 7) / 8), dim3(256), 0,
                        st, static_cast<const __nv_bfloat16*>(x), T, K, (int)D.d, (int)D.R,
                        static_cast<const int32_t*>(slot_of), static_cast<uint8_t*>(x_perm),
                        x_perm_scale);
  // bulk-copy gather: a few CTAs per SM, each streaming its tokens' rows
  const int row_bytes = (int)(D.d * D.x_esz);
  const size_t gsmem = perm::gather_smem_bytes(row_bytes);
  if (gsmem > (size_t)kMaxSmem) return MOE_ERR_UNSUPPORTED;
  int sms = 0;
  moe_status rc2 = device_setup(&sms);
  if (rc2 != MOE_OK) return rc2;
  const int per_sm = (int)(200 * 1024 / gsmem) > 0 ? (int)(200 * 1024 / gsmem) : 1;
  const int grid = T < sms * per_sm ? T : sms * per_sm;
  return launch_chain("k_gather", perm::k_gather, dim3(grid), dim3(32), gsmem, st,
                      static_cast<const uint8_t*>(x), T, K, row_bytes,
                      static_cast<const int32_t*>(slot_of), static_cast<uint8_t*>(x_perm));
}

// FP8 experts: E4M3 x_perm / H with fp32 1x128 scales, E4M3 weights with fp32
// 128x128 block scales, promotion to fp32 every 128 elements of K.
moe_status do_grouped_fp8(const Dims& D, const Layout& L, const void* x_perm,
                          const float* x_perm_scale, const int32_t* gtab, const int32_t* pair_of,
                          const float* topk_w, const void* w_gu, const float* w_gu_scale,
                          const void* w_down, const float* w_down_scale, void* y_slots,
                          uint8_t* ws, int sms, cudaStream_t st) {
  const int E = (int)D.E;
  if (D.d % gemm8::BN) return MOE_ERR_UNSUPPORTED;
  uint8_t* hq = ws + L.hbuf;
  float* hs = reinterpret_cast<float*>(ws + L.hscale);
  const int64_t hrows = D.R + D.Ks * D.T;
  const int64_t mt_bound = (D.R + (int64_t)D.N * 127) / 128 + D.Ks * ((D.T + 127) / 128);
  int stages = 0;
  for (int s = 6; s >= 2 && !stages; --s)
    if (gemm8::smem_bytes(s, E) <= (size_t)kMaxSmem) stages = s;
  if (!stages) return MOE_ERR_UNSUPPORTED;
  const size_t smem = gemm8::smem_bytes(stages, E);
  moe_status rc;
  {
    CUtensorMap ta, tb;
    rc = make_tmap(&ta, x_perm, 1, D.d, D.R + D.T, gemm8::BM);
    if (rc == MOE_OK) rc = make_tmap(&tb, w_gu, 1, D.d, (uint64_t)E * 2 * D.I, 32);
    if (rc != MOE_OK) return rc;
    gemm8::Args a;
    memset(&a, 0, sizeof(a));
    a.gt.base = gtab;
    a.gt.n = E;
    a.n_tiles_n = (int)(D.I / 128);
    a.num_kb = (int)(D.d / 128);
    a.kb_elems = 128;
    a.b_rows_per_expert = (int)(2 * D.I);
    a.b_up_off = (int)D.I;
    a.stages = stages;
    a.idesc = umma_idesc(0, gemm8::BM, gemm8::BN);
    a.a_scale = x_perm_scale;
    a.a_rows = (int)(D.R + D.T);
    a.b_scale = w_gu_scale;
    a.hq = hq;
    a.hs = hs;
    a.inter = (int)D.I;
    const int64_t tiles = mt_bound * a.n_tiles_n;
    const int grid = (int)(tiles < sms ? tiles : sms);
    rc = launch_chain("FP8 grouped GEMM 1", gemm8::k_gemm_promoted<2, gemm8::EPI_SWIGLU_Q>,
                      dim3(grid), dim3(gemm8::NUM_THREADS), smem, st, ta, tb, a);
    if (rc != MOE_OK) return rc;
    if ((rc = trace(3, st)) != MOE_OK) return rc;
  }
  {
    CUtensorMap ta, tb;
    rc = make_tmap(&ta, hq, 1, D.I, hrows, gemm8::BM);
    if (rc == MOE_OK) rc = make_tmap(&tb, w_down, 1, D.I, (uint64_t)E * D.d, gemm8::BN);
    if (rc != MOE_OK) return rc;
    gemm8::Args a;
    memset(&a, 0, sizeof(a));
    a.gt.base = gtab;
    a.gt.n = E;
    a.n_tiles_n = (int)(D.d / gemm8::BN);
    a.num_kb = (int)(D.I / 128);
    a.kb_elems = 128;
    a.b_rows_per_expert = (int)D.d;
    a.a_from_crow = 1;
    a.stages = stages;
    a.idesc = umma_idesc(0, gemm8::BM, gemm8::BN);
    a.a_scale = hs;
    a.a_rows = (int)hrows;
    a.b_scale = w_down_scale;
    a.y = static_cast<__nv_bfloat16*>(y_slots);
    a.d = (int)D.d;
    a.pair_of = pair_of;
    a.topk_w = topk_w;
    a.K = (int)D.K;
    a.Ks = (int)D.Ks;
    const int64_t tiles = mt_bound * a.n_tiles_n;
    const int grid = (int)(tiles < sms ? tiles : sms);
    rc = launch_chain("FP8 grouped GEMM 2", gemm8::k_gemm_promoted<2, gemm8::EPI_SCATTER>,
                      dim3(grid), dim3(gemm8::NUM_THREADS), smem, st, ta, tb, a);
    if (rc != MOE_OK) return rc;
    rc = trace(4, st);
  }
  return rc;
}

// Down projection on 2-CTA clusters: each pair covers 256 W_down rows x up to
// 256 tokens; the grid is the number of clusters that fit at once, times two.
// Launch configuration of a 2-CTA cluster kernel: the grid is the number of
// clusters that fit at once (queried once per kernel and shared-memory size),
// capped by the tile count, times two.
template <typename F>
moe_status pair_config(int slot, F* func, int threads, size_t smem, int64_t tiles,
                       cudaStream_t st, cudaLaunchConfig_t* cfg, cudaLaunchAttribute* attr) {
  memset(cfg, 0, sizeof(*cfg));
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg->blockDim = dim3(threads, 1, 1);
  cfg->dynamicSmemBytes = smem;
  cfg->stream = st;
  cfg->attrs = attr;
  cfg->numAttrs = 1;   // the occupancy query takes the cluster shape only
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int clusters = 0;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo& di = g_dev[dev];
    if (di.pair_smem[slot] != smem) {
      cfg->gridDim = dim3(2 * di.sms, 1, 1);
      e = cudaOccupancyMaxActiveClusters(&clusters, func, cfg);
      if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters");
      di.pair_smem[slot] = smem;
      di.pair_clusters[slot] = clusters;
    }
    clusters = di.pair_clusters[slot];
  }
  if (clusters < 1) return MOE_ERR_UNSUPPORTED;
  if (tiles < clusters) clusters = (int)tiles;
  if (clusters < 1) clusters = 1;
  cfg->gridDim = dim3(2 * clusters, 1, 1);
  cfg->numAttrs = 2;
  return MOE_OK;
}

// n_experts: experts held in w_down (the weight map's extent; the group count
// can be larger or smaller than it).
moe_status launch_down(int kind, const void* w_down, int64_t n_experts, const void* hbuf,
                       size_t esz, int64_t hrows, int64_t tok_tiles, gemmt::Args a,
                       cudaStream_t st) {
  CUtensorMap tw, th;
  moe_status rc = make_tmap(&tw, w_down, esz, a.num_kb * (uint64_t)a.kb_elems,
                            (uint64_t)n_experts * a.w_rows_per_expert, gemmt::WM);
  if (rc == MOE_OK)
    rc = make_tmap(&th, hbuf, esz, a.num_kb * (uint64_t)a.kb_elems, hrows, gemmt::TN / 2);
  if (rc != MOE_OK) return rc;
  int stages = 0;
  for (int s = 8; s >= 2 && !stages; --s)
    if (gemmt::smem_bytes(s, a.gt.n) <= (size_t)kMaxSmem) stages = s;
  if (!stages) return MOE_ERR_UNSUPPORTED;
  a.stages = stages;
  const size_t smem = gemmt::smem_bytes(stages, a.gt.n);
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  rc = kind == 0 ? pair_config(1, gemmt::k_down_gemm<0>, gemmt::NUM_THREADS, smem,
                               tok_tiles * a.n_wt, st, &cfg, attr)
                 : pair_config(1, gemmt::k_down_gemm<1>, gemmt::NUM_THREADS, smem,
                               tok_tiles * a.n_wt, st, &cfg, attr);
  if (rc != MOE_OK) return rc;
  const cudaError_t e = kind == 0 ? cudaLaunchKernelEx(&cfg, gemmt::k_down_gemm<0>, tw, th, a)
                                  : cudaLaunchKernelEx(&cfg, gemmt::k_down_gemm<1>, tw, th, a);
  if (e != cudaSuccess) return cuda_fail(e, "down-projection GEMM (CTA pairs)");
  return launched("down-projection GEMM (CTA pairs)");
}

// Gate/up GEMM with the SwiGLU epilogue on CTA pairs: 128 features x up to
// 256 tokens per cluster tile; shared experts read x, routed experts x_perm.
moe_status launch_gate_up(int kind, const void* w_gu, int64_t n_experts, const void* x,
                          const void* x_perm, size_t esz, int64_t T, int64_t R,
                          int64_t tok_tiles, gemmgu::Args a, cudaStream_t st) {
  const uint64_t inner = a.num_kb * (uint64_t)a.kb_elems;
  CUtensorMap tw, tx, txp;
  moe_status rc = make_tmap(&tw, w_gu, esz, inner, (uint64_t)n_experts * a.w_rows_per_expert,
                            gemmgu::FM);
  if (rc == MOE_OK) rc = make_tmap(&tx, x, esz, inner, T, gemmgu::TN / 2);
  if (rc == MOE_OK) rc = make_tmap(&txp, x_perm, esz, inner, R, gemmgu::TN / 2);
  if (rc != MOE_OK) return rc;
  int stages = 0;
  for (int s = 8; s >= 2 && !stages; --s)
    if (gemmgu::smem_bytes(s, a.gt.n) <= (size_t)kMaxSmem) stages = s;
  if (!stages) return MOE_ERR_UNSUPPORTED;
  a.stages = stages;
  const size_t smem = gemmgu::smem_bytes(stages, a.gt.n);
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  rc = kind == 0 ? pair_config(0, gemmgu::k_gate_up_gemm<0>, gemmgu::NUM_THREADS, smem,
                               tok_tiles * a.n_ft, st, &cfg, attr)
                 : pair_config(0, gemmgu::k_gate_up_gemm<1>, gemmgu::NUM_THREADS, smem,
                               tok_tiles * a.n_ft, st, &cfg, attr);
  if (rc != MOE_OK) return rc;
  const cudaError_t e =
      kind == 0 ? cudaLaunchKernelEx(&cfg, gemmgu::k_gate_up_gemm<0>, tw, tx, txp, a)
                : cudaLaunchKernelEx(&cfg, gemmgu::k_gate_up_gemm<1>, tw, tx, txp, a);
  if (e != cudaSuccess) return cuda_fail(e, "gate/up GEMM (CTA pairs)");
  return launched("gate/up GEMM (CTA pairs)");
}

moe_status do_grouped(const Dims& D, const Layout& L, const void* x, const void* x_perm,
                      const float* x_perm_scale, const int32_t* offsets, const int32_t* slot_of,
                      const float* topk_w, const void* w_gu, const float* w_gu_scale,
                      const void* w_down, const float* w_down_scale, void* y_slots, uint8_t* ws,
                      int sms, cudaStream_t st, __nv_bfloat16* ab_save = nullptr) {
  if (D.T == 0) return MOE_OK;
  const int E = (int)D.E;
  int32_t* gtab = reinterpret_cast<int32_t*>(ws + L.gtab);
  int32_t* pair_of = reinterpret_cast<int32_t*>(ws + L.pair_of);
  void* hbuf = ws + L.hbuf;
  const int prep_blocks = 1 + (int)((D.R + 1023) / 1024 < 4 * sms ? (D.R + 1023) / 1024 : 4 * sms);
  moe_status rc = trace(2, st);
  if (rc != MOE_OK) return rc;
  rc = launch_chain("k_prep_groups", perm::k_prep_groups, dim3(prep_blocks), dim3(1024), 0, st,
                    offsets, (int)D.T, (int)D.K, (int)D.Ks, (int)D.N, D.fp8 ? 1 : 0, gtab,
                    slot_of, pair_of);
  if (rc != MOE_OK) return rc;
  if (D.fp8)
    return do_grouped_fp8(D, L, x_perm, x_perm_scale, gtab, pair_of, topk_w, w_gu, w_gu_scale,
                          w_down, w_down_scale, y_slots, ws, sms, st);

  const size_t esz = D.op_esz;
  const int kind = D.f32 ? 1 : 0;
  const uint32_t fmt = D.f32 ? 2u : 1u;
  const int kbe = (int)(gemm::KB / esz);
  const int64_t hrows = D.R + D.Ks * D.T;
  // upper bound on 256-token tiles over all groups
  const int64_t tok_tiles = (D.R + (int64_t)D.N * 255) / 256 + D.Ks * ((D.T + 255) / 256);

  // GEMM1: H = SiLU(X Wg^T) * (X Wu^T) on CTA pairs: W_gate / W_up rows on the
  // UMMA M side (64 features of each per CTA), up to 256 tokens per tile, so an
  // expert's token tail costs at most 31 padded columns
  {
    gemmgu::Args a;
    memset(&a, 0, sizeof(a));
    a.gt.base = gtab;
    a.gt.n = E;
    a.n_ft = (int)((D.I + 2 * gemmgu::FM - 1) / (2 * gemmgu::FM));
    a.num_kb = (int)(D.d * esz / gemm::KB);
    a.kb_elems = kbe;
    a.inter = (int)D.I;
    a.w_rows_per_expert = (int)(2 * D.I);
    a.fmt = fmt;
    a.out_bf16 = D.f32 ? 0 : 1;
    a.h = hbuf;
    a.ab = ab_save;
    rc = launch_gate_up(kind, w_gu, D.E, x, x_perm, esz, D.T, D.R, tok_tiles, a, st);
    if (rc != MOE_OK) return rc;
    if ((rc = trace(3, st)) != MOE_OK) return rc;
  }
  // GEMM2: Y = H Wd^T, times g, scattered to the token-major slots; W_down rows
  // on the UMMA M side (256 per CTA pair) and up to 256 tokens per tile, so an
  // expert's token tail costs at most 31 padded columns
  {
    gemmt::Args a;
    memset(&a, 0, sizeof(a));
    a.gt.base = gtab;
    a.gt.n = E;
    a.n_wt = (int)((D.d + 2 * gemmt::WM - 1) / (2 * gemmt::WM));
    a.num_kb = (int)(D.I * esz / gemm::KB);
    a.kb_elems = kbe;
    a.w_rows_per_expert = (int)D.d;
    a.fmt = fmt;
    a.out_bf16 = D.f32 ? 0 : 1;
    a.y = y_slots;
    a.d = (int)D.d;
    a.pair_of = pair_of;
    a.topk_w = topk_w;
    a.K = (int)D.K;
    a.Ks = (int)D.Ks;
    rc = launch_down(kind, w_down, D.E, hbuf, esz, hrows, tok_tiles, a, st);
    if (rc != MOE_OK) return rc;
    rc = trace(4, st);
  }
  return rc;
}

moe_status do_combine(const Dims& D, const void* x_res, const void* y, void* h, cudaStream_t st) {
  if (D.T == 0) return MOE_OK;
  const int vec = D.f32 ? 4 : 8;
  const int64_t threads = D.T * (D.d / vec);
  const int blocks = (int)((threads + 255) / 256);
  if (D.f32)
    return launch_chain("k_combine", perm::k_combine<false>, dim3(blocks), dim3(256), 0, st, x_res,
                        y, h, (int)D.T, (int)D.d, (int)D.K, (int)D.Ks);
  return launch_chain("k_combine", perm::k_combine<true>, dim3(blocks), dim3(256), 0, st, x_res,
                      y, h, (int)D.T, (int)D.d, (int)D.K, (int)D.Ks);
}

// ----------------------------------------------------------------------------- expert parallelism
// Workspace of moe_expert_ffn: the group table, then H [n_rows_out, I].
struct FfnLayout {
  size_t gtab, hbuf, hscale, total;
};
FfnLayout ffn_layout(const Dims& D, int n_groups, int64_t n_rows_out) {
  FfnLayout F;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, kAlign); return at; };
  const size_t rows = (size_t)(n_rows_out > 0 ? n_rows_out : 1);
  F.gtab = take((size_t)gemm::group_tab_ints(n_groups) * 4);
  F.hbuf = take(rows * D.I * D.op_esz);
  F.hscale = D.fp8 ? take(rows * (D.I / 128) * 4) : 0;   // E4M3 H: its 1x128 tile scales
  F.total = o;
  return F;
}

// moe_expert_ffn for E4M3 layers: the FP8 grouped GEMMs over caller-given row
// groups (x_rows codes and 1x128 scales in, H requantised per 1x128 between
// the GEMMs, bf16 rows out in plain-row mode).
moe_status do_expert_ffn_fp8(const Dims& D, int n_experts, int n_groups, const int32_t* groups,
                             int64_t n_in, int64_t n_out, const void* x_rows,
                             const float* x_rows_scale, const float* row_w, const void* w_gu,
                             const float* w_gu_scale, const void* w_down,
                             const float* w_down_scale, void* y_rows, const uint64_t* group_out,
                             uint8_t* ws, int sms, cudaStream_t st) {
  if (D.d % gemm8::BN || D.I % 128) return MOE_ERR_UNSUPPORTED;
  const FfnLayout F = ffn_layout(D, n_groups, n_out);
  int32_t* gtab = reinterpret_cast<int32_t*>(ws + F.gtab);
  uint8_t* hq = ws + F.hbuf;
  float* hs = reinterpret_cast<float*>(ws + F.hscale);
  moe_status rc = launch_chain("k_prep_user_groups", perm::k_prep_user_groups, dim3(1),
                               dim3(1024), 0, st, groups, n_groups, n_experts, (int)n_in,
                               (int)n_out, gtab);
  if (rc != MOE_OK) return rc;
  int stages = 0;
  for (int s = 6; s >= 2 && !stages; --s)
    if (gemm8::smem_bytes(s, n_groups) <= (size_t)kMaxSmem) stages = s;
  if (!stages) return MOE_ERR_UNSUPPORTED;
  const size_t smem = gemm8::smem_bytes(stages, n_groups);
  // upper bound on 128-row tiles over all groups
  const int64_t mt_bound = (n_out + (int64_t)n_groups * 127) / 128;
  {
    CUtensorMap ta, tb;
    rc = make_tmap(&ta, x_rows, 1, D.d, (uint64_t)n_in, gemm8::BM);
    if (rc == MOE_OK) rc = make_tmap(&tb, w_gu, 1, D.d, (uint64_t)n_experts * 2 * D.I, 32);
    if (rc != MOE_OK) return rc;
    gemm8::Args a;
    memset(&a, 0, sizeof(a));
    a.gt.base = gtab;
    a.gt.n = n_groups;
    a.n_tiles_n = (int)(D.I / 128);
    a.num_kb = (int)(D.d / 128);
    a.kb_elems = 128;
    a.b_rows_per_expert = (int)(2 * D.I);
    a.b_up_off = (int)D.I;
    a.stages = stages;
    a.idesc = umma_idesc(0, gemm8::BM, gemm8::BN);
    a.a_scale = x_rows_scale;
    a.a_rows = (int)n_in;
    a.b_scale = w_gu_scale;
    a.hq = hq;
    a.hs = hs;
    a.inter = (int)D.I;
    const int64_t tiles = mt_bound * a.n_tiles_n;
    const int grid = (int)(tiles < sms ? tiles : sms);
    rc = launch_chain("FP8 expert GEMM 1", gemm8::k_gemm_promoted<2, gemm8::EPI_SWIGLU_Q>,
                      dim3(grid), dim3(gemm8::NUM_THREADS), smem, st, ta, tb, a);
    if (rc != MOE_OK) return rc;
  }
  {
    CUtensorMap ta, tb;
    rc = make_tmap(&ta, hq, 1, D.I, (uint64_t)n_out, gemm8::BM);
    if (rc == MOE_OK) rc = make_tmap(&tb, w_down, 1, D.I, (uint64_t)n_experts * D.d, gemm8::BN);
    if (rc != MOE_OK) return rc;
    gemm8::Args a;
    memset(&a, 0, sizeof(a));
    a.gt.base = gtab;
    a.gt.n = n_groups;
    a.n_tiles_n = (int)(D.d / gemm8::BN);
    a.num_kb = (int)(D.I / 128);
    a.kb_elems = 128;
    a.b_rows_per_expert = (int)D.d;
    a.a_from_crow = 1;
    a.stages = stages;
    a.idesc = umma_idesc(0, gemm8::BM, gemm8::BN);
    a.a_scale = hs;
    a.a_rows = (int)n_out;
    a.b_scale = w_down_scale;
    a.y = static_cast<__nv_bfloat16*>(y_rows);
    a.d = (int)D.d;
    a.plain = 1;
    a.row_w = row_w;
    a.group_base = reinterpret_cast<const unsigned long long*>(group_out);
    const int64_t tiles = mt_bound * a.n_tiles_n;
    const int grid = (int)(tiles < sms ? tiles : sms);
    rc = launch_chain("FP8 expert GEMM 2", gemm8::k_gemm_promoted<2, gemm8::EPI_SCATTER>,
                      dim3(grid), dim3(gemm8::NUM_THREADS), smem, st, ta, tb, a);
  }
  return rc;
}

moe_status do_expert_ffn(const Dims& D, int n_experts, int n_groups, const int32_t* groups,
                         int64_t n_in, int64_t n_out, const void* x_rows, const float* row_w,
                         const void* w_gu, const void* w_down, void* y_rows,
                         const uint64_t* group_out, uint8_t* ws, int sms, cudaStream_t st) {
  const FfnLayout F = ffn_layout(D, n_groups, n_out);
  int32_t* gtab = reinterpret_cast<int32_t*>(ws + F.gtab);
  void* hbuf = ws + F.hbuf;
  moe_status rc = launch_chain("k_prep_user_groups", perm::k_prep_user_groups, dim3(1),
                               dim3(1024), 0, st, groups, n_groups, n_experts, (int)n_in,
                               (int)n_out, gtab);
  if (rc != MOE_OK) return rc;
  const size_t esz = D.op_esz;
  const int kind = D.f32 ? 1 : 0;
  const uint32_t fmt = D.f32 ? 2u : 1u;
  const int kbe = (int)(gemm::KB / esz);
  // upper bound on 256-token tiles over all groups
  const int64_t tok_tiles = (n_out + (int64_t)n_groups * 255) / 256;
  {
    gemmgu::Args a;
    memset(&a, 0, sizeof(a));
    a.gt.base = gtab;
    a.gt.n = n_groups;
    a.n_ft = (int)((D.I + 2 * gemmgu::FM - 1) / (2 * gemmgu::FM));
    a.num_kb = (int)(D.d * esz / gemm::KB);
    a.kb_elems = kbe;
    a.inter = (int)D.I;
    a.w_rows_per_expert = (int)(2 * D.I);
    a.fmt = fmt;
    a.out_bf16 = D.f32 ? 0 : 1;
    a.h = hbuf;
    rc = launch_gate_up(kind, w_gu, n_experts, x_rows, x_rows, esz, n_in, n_in, tok_tiles, a,
                        st);
    if (rc != MOE_OK) return rc;
  }
  {
    gemmt::Args a;
    memset(&a, 0, sizeof(a));
    a.gt.base = gtab;
    a.gt.n = n_groups;
    a.n_wt = (int)((D.d + 2 * gemmt::WM - 1) / (2 * gemmt::WM));
    a.num_kb = (int)(D.I * esz / gemm::KB);
    a.kb_elems = kbe;
    a.w_rows_per_expert = (int)D.d;
    a.fmt = fmt;
    a.out_bf16 = D.f32 ? 0 : 1;
    a.y = y_rows;
    a.d = (int)D.d;
    a.plain = 1;
    a.row_w = row_w;
    a.group_base = reinterpret_cast<const unsigned long long*>(group_out);
    rc = launch_down(kind, w_down, n_experts, hbuf, esz, n_out, tok_tiles, a, st);
  }
  return rc;
}

// ----------------------------------------------------------------------------- backward
// Workspace of moe_backward: the forward's routing buffers (same offsets as
// the forward layout), then the padded row buffers of the backward.
struct BwdLayout {
  size_t poff, tabs, row_pair, row_w, x_pad, dh_pad, ab, dab, zg, dgp, dl, dxr, dslots, total;
  int64_t rows_routed;   // rows of x_pad / dh_pad (routed segments, padded)
  int64_t rows;          // rows of ab / dab / zg / dgp (routed and shared segments)
  int n_it;              // feature tiles of 256 over I (partials per row)
};

constexpr int kBwdTables = 7;

BwdLayout bwd_layout(const Dims& D, const Layout& L) {
  BwdLayout B;
  size_t o = align_up(L.gtab + (size_t)gemm::group_tab_ints((int)D.E) * 4, kAlign);
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, kAlign); return at; };
  B.rows_routed = D.R + (int64_t)bwd::PAD * D.N;
  B.rows = B.rows_routed + D.Ks * (int64_t)bwd::pad64((int)D.T);
  B.n_it = (int)((D.I + gbwd::BN - 1) / gbwd::BN);
  B.poff = take((size_t)(D.E + 1) * 4);
  B.tabs = take((size_t)kBwdTables * D.E * gbwd::GB_FIELDS * 4);
  B.row_pair = take((size_t)B.rows * 4);
  B.row_w = take((size_t)B.rows * 4);
  B.x_pad = take((size_t)B.rows_routed * D.d * 2);
  B.dh_pad = take((size_t)B.rows_routed * D.d * 2);
  B.ab = take((size_t)B.rows * 2 * D.I * 2);
  B.dab = take((size_t)B.rows * 2 * D.I * 2);
  B.zg = take((size_t)B.rows * D.I * 2);
  B.dgp = take((size_t)B.rows * B.n_it * 4);
  B.dl = take((size_t)D.T * D.N * 2);
  B.dxr = take((size_t)D.T * D.d * 2);
  B.dslots = take((size_t)D.T * (D.K + D.Ks) * D.d * 2);
  B.total = o;
  return B;
}

// 2-D tensor map for an operand read MN-major: rows of `inner` bf16 elements
// (the M or N extent), `rows` rows (the K extent); box = 64 elements x 64 rows.
moe_status make_tmap_mn(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows) {
  cuuint64_t dims[2] = {inner, rows > 0 ? rows : 1};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(t_errmsg, sizeof(t_errmsg), "cuTensorMapEncodeTiled (MN-major): CUresult %d "
             "(rows %llu, inner %llu)", (int)r, (unsigned long long)rows,
             (unsigned long long)inner);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// One operand of a backward GEMM: base, row length and row count, and whether
// it is read MN-major (its rows are the K index).
struct Operand {
  const void* base;
  uint64_t inner, rows;
};

// The activation-side backward problems (A = token rows, K-major) on CTA
// pairs: 256-row tiles, each CTA loading its 128 rows and half of the tile's
// 256 B columns.
template <bool B_MN, int EPI>
moe_status launch_gemm_bwd(const char* what, Operand a0, Operand a1, Operand b0, Operand b1,
                           gbwd::Args args, int64_t tiles_bound, cudaStream_t st) {
  CUtensorMap ta0, ta1, tb0, tb1;
  auto mk = [&](CUtensorMap* m, const Operand& o, bool mn, uint32_t box_rows) {
    return mn ? make_tmap_mn(m, o.base, o.inner, o.rows) : make_tmap(m, o.base, 2, o.inner, o.rows,
                                                                     box_rows);
  };
  moe_status rc = mk(&ta0, a0, false, gbwd::BM);
  if (rc == MOE_OK) rc = mk(&ta1, a1, false, gbwd::BM);
  if (rc == MOE_OK) rc = mk(&tb0, b0, B_MN, gbwd::BN / 2);
  if (rc == MOE_OK) rc = mk(&tb1, b1, B_MN, gbwd::BN / 2);
  if (rc != MOE_OK) return rc;
  int stages = 0;
  for (int s = 6; s >= 2 && !stages; --s)
    if (gbwd::smem_bytes(s, args.n_probs) <= (size_t)kMaxSmem) stages = s;
  if (!stages) return MOE_ERR_UNSUPPORTED;
  args.stages = stages;
  const size_t smem = gbwd::smem_bytes(stages, args.n_probs);
  auto* k = gbwd::k_gemm_bwd<B_MN, EPI>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  if (e != cudaSuccess) return cuda_fail(e, what);
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  rc = pair_config(3, k, gbwd::NUM_THREADS, smem, tiles_bound, st, &cfg, attr);
  if (rc != MOE_OK) return rc;
  e = cudaLaunchKernelEx(&cfg, k, ta0, ta1, tb0, tb1, args);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return launched(what);
}

// Output map of the weight-gradient GEMMs: fp32 or bf16 [nz][m][ldc], box
// 32 x 32 x 1; fp32 with the 128-byte swizzle, bf16 unswizzled (the
// epilogue's staging layouts).  Rows are one expert's,
// so a TMA store clips at the expert's last row and at the row's end.
moe_status make_tmap_out(CUtensorMap* mp, void* base, uint64_t ldc, uint64_t m, uint64_t nz,
                         bool bf16) {
  const uint64_t esz = bf16 ? 2 : 4;
  if ((ldc * esz) % 16 != 0 || m == 0 || nz == 0) {
    snprintf(t_errmsg, sizeof(t_errmsg), "weight-gradient output map: rows of %llu elements "
             "are not a multiple of 16 bytes", (unsigned long long)ldc);
    return MOE_ERR_UNSUPPORTED;
  }
  cuuint64_t dims[3] = {ldc, m, nz};
  cuuint64_t strides[2] = {ldc * esz, m * ldc * esz};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(mp, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                        3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        bf16 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(t_errmsg, sizeof(t_errmsg), "cuTensorMapEncodeTiled (gradient output): CUresult %d "
             "(row %llu, rows %llu, experts %llu)", (int)r, (unsigned long long)ldc,
             (unsigned long long)m, (unsigned long long)nz);
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// The weight-gradient problems on CTA pairs (k_gemm_bwd_pair): 256 x 256 pair
// tiles, grid = co-resident pairs (capped by the tile count) x 2.  Every
// problem's output is the expert's block crow = e * m_rows of args.c with N =
// args.ldc columns; the epilogue stores through a [n_z][m_rows][ldc] map.
moe_status launch_gemm_bwd_pair(const char* what, Operand a0, Operand a1, Operand b0, Operand b1,
                                gbwd::Args args, uint64_t m_rows, uint64_t n_z,
                                int64_t pair_tiles_bound, bool bf16_out, cudaStream_t st) {
  CUtensorMap ta0, ta1, tb0, tb1, tc;
  moe_status rc = make_tmap_mn(&ta0, a0.base, a0.inner, a0.rows);
  if (rc == MOE_OK) rc = make_tmap_mn(&ta1, a1.base, a1.inner, a1.rows);
  if (rc == MOE_OK) rc = make_tmap_mn(&tb0, b0.base, b0.inner, b0.rows);
  if (rc == MOE_OK) rc = make_tmap_mn(&tb1, b1.base, b1.inner, b1.rows);
  if (rc == MOE_OK) rc = make_tmap_out(&tc, args.c, (uint64_t)args.ldc, m_rows, n_z, bf16_out);
  if (rc != MOE_OK) return rc;
  int stages = 0;
  for (int s = 6; s >= 2 && !stages; --s)
    if (gbwd::pair_smem_bytes(s, args.n_probs) <= (size_t)kMaxSmem) stages = s;
  if (!stages) return MOE_ERR_UNSUPPORTED;
  args.stages = stages;
  const size_t smem = gbwd::pair_smem_bytes(stages, args.n_probs);
  auto* k = bf16_out ? gbwd::k_gemm_bwd_pair<true> : gbwd::k_gemm_bwd_pair<false>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  if (e != cudaSuccess) return cuda_fail(e, what);
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  rc = pair_config(2, k, gbwd::NUM_THREADS, smem, pair_tiles_bound, st, &cfg, attr);
  if (rc != MOE_OK) return rc;
  e = cudaLaunchKernelEx(&cfg, k, ta0, ta1, tb0, tb1, tc, args);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return launched(what);
}

template <int VPL>
moe_status launch_gate_bwd(const float* logits, const route::Params& p, const int32_t* idx,
                           const int32_t* slot_of, const int32_t* offsets, const int32_t* poff,
                           const float* dgp, int n_it, __nv_bfloat16* dl, cudaStream_t st) {
  return launch_chain("k_gate_bwd", bwd::k_gate_bwd<VPL>, dim3((p.T + 7) / 8), dim3(256), 0, st,
                      logits, p, idx, slot_of, offsets, poff, dgp, n_it, dl);
}

moe_status do_backward(const moe_layer_desc& s, const Dims& D, const Layout& L,
                       const BwdLayout& B, const void* x, const void* w_router,
                       const float* bias, const void* w_gu, const void* w_down, const void* dh,
                       void* dx, void* dw_router, void* dw_gu, void* dw_down, bool bf16_grads,
                       const void* ab_saved, uint8_t* ws, int sms, cudaStream_t st) {
  const int T = (int)D.T, d = (int)D.d, I = (int)D.I, N = (int)D.N, K = (int)D.K;
  const int Ks = (int)D.Ks, E = (int)D.E;
  int32_t* idx = reinterpret_cast<int32_t*>(ws + L.topk_idx);
  float* tw = reinterpret_cast<float*>(ws + L.topk_w);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + L.hist);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* perm_src = reinterpret_cast<int32_t*>(ws + L.perm_src);
  int32_t* slot_of = reinterpret_cast<int32_t*>(ws + L.slot_of);
  const float* logits = reinterpret_cast<const float*>(ws + L.logits);
  int32_t* poff = reinterpret_cast<int32_t*>(ws + B.poff);
  int32_t* tabs = reinterpret_cast<int32_t*>(ws + B.tabs);
  const size_t tab_ints = (size_t)E * gbwd::GB_FIELDS;
  int32_t* tab[kBwdTables];
  for (int i = 0; i < kBwdTables; ++i) tab[i] = tabs + i * tab_ints;
  int32_t* row_pair = reinterpret_cast<int32_t*>(ws + B.row_pair);
  float* row_w = reinterpret_cast<float*>(ws + B.row_w);
  auto* x_pad = reinterpret_cast<__nv_bfloat16*>(ws + B.x_pad);
  auto* dh_pad = reinterpret_cast<__nv_bfloat16*>(ws + B.dh_pad);
  auto* ab = reinterpret_cast<__nv_bfloat16*>(ws + B.ab);
  auto* dab = reinterpret_cast<__nv_bfloat16*>(ws + B.dab);
  auto* zg = reinterpret_cast<__nv_bfloat16*>(ws + B.zg);
  float* dgp = reinterpret_cast<float*>(ws + B.dgp);
  auto* dl = reinterpret_cast<__nv_bfloat16*>(ws + B.dl);
  auto* dxr = reinterpret_cast<__nv_bfloat16*>(ws + B.dxr);
  auto* dslots = reinterpret_cast<__nv_bfloat16*>(ws + B.dslots);

  // routing and the permutation maps, as in the forward
  moe_status rc = do_route(s, D, L, x, w_router, bias, idx, tw, nullptr, ws, sms, st);
  if (rc != MOE_OK) return rc;
  rc = launch_chain("k_hist", perm::k_hist, dim3(D.n_chunks), dim3(256), N * 4, st,
                    static_cast<const int32_t*>(idx), T, K, N, hist);
  if (rc == MOE_OK)
    rc = launch_scan(st, hist, (int)D.n_chunks,
                      N, static_cast<const int32_t*>(nullptr), counts, offsets);
  if (rc == MOE_OK)
    rc = launch_chain("k_slots", perm::k_slots, dim3(D.n_chunks), dim3(perm::SLOT_WARPS * 32),
                      perm::SLOT_WARPS * N * 4, st, static_cast<const int32_t*>(idx), T, K, N,
                      static_cast<const int32_t*>(hist), slot_of, perm_src);
  if (rc != MOE_OK) return rc;
  bwd::PrepArgs pa;
  pa.offsets = offsets;
  pa.T = T; pa.d = d; pa.I = I; pa.Ks = Ks; pa.N = N;
  pa.poff = poff;
  pa.tab_ab = tab[0]; pa.tab_dz = tab[1]; pa.tab_du = tab[2]; pa.tab_dwd = tab[3];
  pa.tab_dwgu = tab[4]; pa.tab_dxr = tab[5]; pa.tab_dwr = tab[6];
  rc = launch_chain("k_bwd_prep", bwd::k_bwd_prep, dim3(1), dim3(1024), 0, st, pa);
  if (rc == MOE_OK)
    rc = launch_chain("k_bwd_gather", bwd::k_bwd_gather, dim3((T + 7) / 8), dim3(256), 0, st,
                      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(dh),
                      T, K, d, static_cast<const int32_t*>(idx), static_cast<const float*>(tw),
                      static_cast<const int32_t*>(slot_of), static_cast<const int32_t*>(offsets),
                      static_cast<const int32_t*>(poff), N, x_pad, dh_pad, row_pair, row_w);
  if (rc == MOE_OK)
    rc = launch_chain("k_bwd_zero_pads", bwd::k_bwd_zero_pads, dim3(N), dim3(256), 0, st,
                      static_cast<const int32_t*>(offsets), static_cast<const int32_t*>(poff), d,
                      x_pad, dh_pad, row_pair, row_w);
  if (rc != MOE_OK) return rc;

  // tile bounds for the grid size (the exact counts are known on the device only)
  const int64_t mt_rows = (B.rows + gbwd::BM - 1) / gbwd::BM + E;
  auto nt = [](int64_t n) { return (n + gbwd::BN - 1) / gbwd::BN; };
  const uint64_t W_gu_rows = (uint64_t)E * 2 * I, W_d_rows = (uint64_t)E * d;
  const Operand X{x, (uint64_t)d, (uint64_t)T}, DH{dh, (uint64_t)d, (uint64_t)T};
  const Operand XP{x_pad, (uint64_t)d, (uint64_t)B.rows_routed};
  const Operand DHP{dh_pad, (uint64_t)d, (uint64_t)B.rows_routed};
  const Operand WGU{w_gu, (uint64_t)d, W_gu_rows}, WD{w_down, (uint64_t)I, W_d_rows};
  const Operand AB{ab, (uint64_t)(2 * I), (uint64_t)B.rows};
  const Operand DAB{dab, (uint64_t)(2 * I), (uint64_t)B.rows};
  const Operand ZG{zg, (uint64_t)I, (uint64_t)B.rows};
  const Operand DL{dl, (uint64_t)N, (uint64_t)T}, WR{w_router, (uint64_t)d, (uint64_t)N};
  (void)AB;
  gbwd::Args ga;
  memset(&ga, 0, sizeof(ga));
  ga.n_probs = E;
  ga.K = K;
  ga.Ks = Ks;
  ga.inter = I;
  // G1: a | b pre-activations of every (row, expert), unless the forward kept them
  if (!ab_saved) {
    ga.tab = tab[0];
    ga.c = ab;
    ga.ldc = 2 * I;
    rc = launch_gemm_bwd<false, gbwd::EPI_BF16>("backward GEMM ab = X W_gu^T", X, XP, WGU, WGU,
                                                ga, mt_rows * nt(2 * I), st);
    if (rc != MOE_OK) return rc;
  }
  // G2: dz' = dY W_down with the SwiGLU backward in the epilogue
  ga.tab = tab[1];
  ga.c = nullptr;
  ga.ab = ab;
  ga.ab_saved = static_cast<const __nv_bfloat16*>(ab_saved);
  ga.zg = zg;
  ga.dab = dab;
  ga.dgp = dgp;
  ga.row_w = row_w;
  rc = launch_gemm_bwd<true, gbwd::EPI_SWIGLU_BWD>("backward GEMM dz = dY W_down", DH, DHP, WD,
                                                   WD, ga, mt_rows * nt(I), st);
  if (rc != MOE_OK) return rc;
  // G3: du pieces = [da | db] W_gu, scattered to the token-major slots
  ga.tab = tab[2];
  ga.c = dslots;
  ga.ldc = d;
  ga.row_pair = row_pair;
  rc = launch_gemm_bwd<true, gbwd::EPI_SCATTER>("backward GEMM du = dAB W_gu", DAB, DAB, WGU,
                                                WGU, ga, mt_rows * nt(d), st);
  if (rc != MOE_OK) return rc;
  // gate-weight and affinity backward -> dl [T, N]
  {
    const route::Params p = route_params(s);
    if (N <= 32) rc = launch_gate_bwd<1>(logits, p, idx, slot_of, offsets, poff, dgp, B.n_it, dl, st);
    else if (N <= 64) rc = launch_gate_bwd<2>(logits, p, idx, slot_of, offsets, poff, dgp, B.n_it, dl, st);
    else if (N <= 128) rc = launch_gate_bwd<4>(logits, p, idx, slot_of, offsets, poff, dgp, B.n_it, dl, st);
    else if (N <= 256) rc = launch_gate_bwd<8>(logits, p, idx, slot_of, offsets, poff, dgp, B.n_it, dl, st);
    else rc = launch_gate_bwd<16>(logits, p, idx, slot_of, offsets, poff, dgp, B.n_it, dl, st);
    if (rc != MOE_OK) return rc;
  }
  // G6a: the router's part of dx, dx_router = dl W_r
  ga.n_probs = 1;
  ga.tab = tab[5];
  ga.c = dxr;
  ga.ldc = d;
  rc = launch_gemm_bwd<true, gbwd::EPI_BF16>("backward GEMM dx_router = dL W_r", DL, DL, WR, WR,
                                             ga, nt(d) * ((T + 127) / 128), st);
  if (rc != MOE_OK) return rc;
  // dx = dx_router + sum over the token's expert slots, fp32, fixed order
  rc = do_combine(D, dxr, dslots, dx, st);
  if (rc != MOE_OK) return rc;
  // G4: dW_down = dY^T (g z) over each expert's rows
  ga.n_probs = E;
  ga.tab = tab[3];
  ga.c = dw_down;
  ga.ldc = I;
  rc = launch_gemm_bwd_pair("backward GEMM dW_down = dY^T Z (CTA pairs)", DH, DHP, ZG, ZG, ga,
                            (uint64_t)d, (uint64_t)E, (int64_t)E * ((d + 255) / 256) * nt(I),
                            bf16_grads, st);
  if (rc != MOE_OK) return rc;
  // G5: dW_gu = [da | db]^T X over each expert's rows
  ga.tab = tab[4];
  ga.c = dw_gu;
  ga.ldc = d;
  rc = launch_gemm_bwd_pair("backward GEMM dW_gu = dAB^T X (CTA pairs)", DAB, DAB, X, XP, ga,
                            (uint64_t)(2 * I), (uint64_t)E,
                            (int64_t)E * ((2 * I + 255) / 256) * nt(d), bf16_grads, st);
  if (rc != MOE_OK) return rc;
  // G6b: dW_r = dl^T X over all tokens
  ga.n_probs = 1;
  ga.tab = tab[6];
  ga.c = dw_router;
  ga.ldc = d;
  return launch_gemm_bwd_pair("backward GEMM dW_r = dL^T X (CTA pairs)", DL, DL, X, X, ga,
                              (uint64_t)N, 1, ((N + 255) / 256) * nt(d), bf16_grads, st);
}

// ----------------------------------------------------------------------------- FP8 backward
// Workspace of moe_backward_fp8: the forward's routing buffers, then the
// 128-padded row space (routed segments, then one per shared expert) and the
// FP8 operands of the backward GEMMs.
struct Bwd8Layout {
  int64_t rs;            // rows of the row space (a bound; a multiple of 128)
  size_t poff, gtab, gtab_wd, gtab_wgu, kgroup, tabs, row_pair, row_w, row_tok;
  size_t xq, xs, dhq, dhs, ab, zg, dab, dgp, dabq, dabs, dl, dxr, dslots;
  size_t dhT, dhTs, zgT, zgTs, dabT, dabTs, xT, xTs, total;
};

Bwd8Layout bwd8_layout(const Dims& D, const Layout& L) {
  Bwd8Layout B;
  size_t o = align_up(L.gtab + (size_t)gemm::group_tab_ints((int)D.E) * 4, kAlign);
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, kAlign); return at; };
  const int64_t rs = (D.R + 127 * D.N + 127) / 128 * 128 + D.Ks * (int64_t)bwd8::pad128((int)D.T);
  const size_t d = D.d, I = D.I, R = (size_t)rs, E = D.E;
  B.rs = rs;
  B.poff = take((E + 1) * 4);
  B.gtab = take((size_t)gemm::group_tab_ints((int)E) * 4);
  B.gtab_wd = take((size_t)gemm::group_tab_ints((int)E) * 4);
  B.gtab_wgu = take((size_t)gemm::group_tab_ints((int)E) * 4);
  B.kgroup = take(2 * E * 4);
  B.tabs = take(2 * gbwd::GB_FIELDS * 4);
  B.row_pair = take(R * 4);
  B.row_w = take(R * 4);
  B.row_tok = take(R * 4);
  B.xq = take(R * d);
  B.xs = take(R * (d / 128) * 4);
  B.dhq = take(R * d);
  B.dhs = take(R * (d / 128) * 4);
  B.ab = take(R * 2 * I * 2);
  B.zg = take(R * I * 2);
  B.dab = take(R * 2 * I * 2);
  B.dgp = take(R * (I / 64) * 4);
  B.dabq = take(R * 2 * I);
  B.dabs = take(R * (2 * I / 128) * 4);
  B.dl = take((size_t)D.T * D.N * 2);
  B.dxr = take((size_t)D.T * d * 2);
  B.dslots = take((size_t)D.T * (D.K + D.Ks) * d * 2);
  B.dhT = take(d * R);
  B.dhTs = take((R / 128) * d * 4);
  B.zgT = take(I * R);
  B.zgTs = take((R / 128) * I * 4);
  B.dabT = take(2 * I * R);
  B.dabTs = take((R / 128) * 2 * I * 4);
  B.xT = take(d * R);
  B.xTs = take((R / 128) * d * 4);
  B.total = o;
  return B;
}

struct Fp8Weights {
  const void *gu, *gu_t, *down_t;
  const float *gu_s, *gu_t_s, *down_t_s;
};

moe_status do_backward_fp8(const moe_layer_desc& s, const Dims& D, const Layout& L,
                           const Bwd8Layout& B, const void* x, const void* w_router,
                           const float* bias, const Fp8Weights& W, const void* dh, void* dx,
                           void* dw_router, void* dw_gu, void* dw_down, uint8_t* ws, int sms,
                           cudaStream_t st) {
  const int T = (int)D.T, d = (int)D.d, I = (int)D.I, N = (int)D.N, K = (int)D.K;
  const int Ks = (int)D.Ks, E = (int)D.E;
  const int rs = (int)B.rs;
  int32_t* idx = reinterpret_cast<int32_t*>(ws + L.topk_idx);
  float* tw = reinterpret_cast<float*>(ws + L.topk_w);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + L.hist);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* perm_src = reinterpret_cast<int32_t*>(ws + L.perm_src);
  int32_t* slot_of = reinterpret_cast<int32_t*>(ws + L.slot_of);
  const float* logits = reinterpret_cast<const float*>(ws + L.logits);
  int32_t* poff = reinterpret_cast<int32_t*>(ws + B.poff);
  int32_t* gtab = reinterpret_cast<int32_t*>(ws + B.gtab);
  int32_t* gtab_wd = reinterpret_cast<int32_t*>(ws + B.gtab_wd);
  int32_t* gtab_wgu = reinterpret_cast<int32_t*>(ws + B.gtab_wgu);
  int32_t* kgroup = reinterpret_cast<int32_t*>(ws + B.kgroup);
  int32_t* tab_dxr = reinterpret_cast<int32_t*>(ws + B.tabs);
  int32_t* tab_dwr = tab_dxr + gbwd::GB_FIELDS;
  int32_t* row_pair = reinterpret_cast<int32_t*>(ws + B.row_pair);
  float* row_w = reinterpret_cast<float*>(ws + B.row_w);
  int32_t* row_tok = reinterpret_cast<int32_t*>(ws + B.row_tok);
  uint8_t* xq = ws + B.xq;
  float* xs = reinterpret_cast<float*>(ws + B.xs);
  uint8_t* dhq = ws + B.dhq;
  float* dhs = reinterpret_cast<float*>(ws + B.dhs);
  auto* ab = reinterpret_cast<__nv_bfloat16*>(ws + B.ab);
  auto* zg = reinterpret_cast<__nv_bfloat16*>(ws + B.zg);
  auto* dab = reinterpret_cast<__nv_bfloat16*>(ws + B.dab);
  float* dgp = reinterpret_cast<float*>(ws + B.dgp);
  uint8_t* dabq = ws + B.dabq;
  float* dabs = reinterpret_cast<float*>(ws + B.dabs);
  auto* dl = reinterpret_cast<__nv_bfloat16*>(ws + B.dl);
  auto* dxr = reinterpret_cast<__nv_bfloat16*>(ws + B.dxr);
  auto* dslots = reinterpret_cast<__nv_bfloat16*>(ws + B.dslots);

  // routing and the permutation maps, as in the forward
  moe_status rc = do_route(s, D, L, x, w_router, bias, idx, tw, nullptr, ws, sms, st);
  if (rc != MOE_OK) return rc;
  rc = launch_chain("k_hist", perm::k_hist, dim3(D.n_chunks), dim3(256), N * 4, st,
                    static_cast<const int32_t*>(idx), T, K, N, hist);
  if (rc == MOE_OK)
    rc = launch_scan(st, hist, (int)D.n_chunks, N, static_cast<const int32_t*>(nullptr), counts,
                     offsets);
  if (rc == MOE_OK)
    rc = launch_chain("k_slots", perm::k_slots, dim3(D.n_chunks), dim3(perm::SLOT_WARPS * 32),
                      perm::SLOT_WARPS * N * 4, st, static_cast<const int32_t*>(idx), T, K, N,
                      static_cast<const int32_t*>(hist), slot_of, perm_src);
  if (rc != MOE_OK) return rc;
  bwd8::PrepArgs pa;
  pa.offsets = offsets;
  pa.T = T; pa.d = d; pa.I = I; pa.Ks = Ks; pa.N = N;
  pa.poff = poff; pa.gtab = gtab; pa.gtab_wd = gtab_wd; pa.gtab_wgu = gtab_wgu;
  pa.kgroup = kgroup; pa.tab_dxr = tab_dxr; pa.tab_dwr = tab_dwr;
  rc = launch_chain("k_bwd8_prep", bwd8::k_bwd8_prep, dim3(1), dim3(1024), 0, st, pa);
  if (rc == MOE_OK)
    rc = launch_chain("k_bwd8_gather", bwd8::k_bwd8_gather, dim3((T + 7) / 8), dim3(256), 0, st,
                      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(dh),
                      T, K, Ks, N, d, static_cast<const int32_t*>(idx),
                      static_cast<const float*>(tw), static_cast<const int32_t*>(slot_of),
                      static_cast<const int32_t*>(offsets), static_cast<const int32_t*>(poff), xq,
                      xs, dhq, dhs, row_pair, row_w, row_tok);
  if (rc == MOE_OK)
    rc = launch_chain("k_bwd8_pads", bwd8::k_bwd8_pads, dim3(E + 1), dim3(128), 0, st,
                      static_cast<const int32_t*>(offsets), N, T, rs,
                      static_cast<const int32_t*>(poff), row_pair, row_w, row_tok);
  if (rc != MOE_OK) return rc;

  int stages = 0, wg_stages = 0;
  for (int sg = 6; sg >= 2 && !stages; --sg)
    if (gemm8::smem_bytes(sg, E) <= (size_t)kMaxSmem) stages = sg;
  for (int sg = 6; sg >= 2 && !wg_stages; --sg)
    if (gemm8::smem_bytes(sg, E, true) <= (size_t)kMaxSmem) wg_stages = sg;
  if (!stages || !wg_stages) return MOE_ERR_UNSUPPORTED;
  const size_t smem = gemm8::smem_bytes(stages, E);
  const size_t wg_smem = gemm8::smem_bytes(wg_stages, E, true);
  const int64_t mt_rows = rs / 128;                  // m-tiles of the row space (a bound)
  auto grid_of = [&](int64_t tiles) { return (int)(tiles < sms ? tiles : sms); };
  auto base_args = [&](const int32_t* gt, int n_tiles_n, int num_kb, int b_rows_per_expert) {
    gemm8::Args a;
    memset(&a, 0, sizeof(a));
    a.gt.base = gt;
    a.gt.n = E;
    a.n_tiles_n = n_tiles_n;
    a.num_kb = num_kb;
    a.kb_elems = 128;
    a.b_rows_per_expert = b_rows_per_expert;
    a.stages = stages;
    a.idesc = umma_idesc(0, gemm8::BM, gemm8::BN);
    a.K = K;
    a.Ks = Ks;
    a.inter = I;
    return a;
  };
  // G1: a | b = X W_gu^T, X rows in FP8
  {
    CUtensorMap ta, tb;
    rc = make_tmap(&ta, xq, 1, d, rs, gemm8::BM);
    if (rc == MOE_OK) rc = make_tmap(&tb, W.gu, 1, d, (uint64_t)E * 2 * I, gemm8::BN);
    if (rc != MOE_OK) return rc;
    gemm8::Args a = base_args(gtab, 2 * I / gemm8::BN, d / 128, 2 * I);
    a.a_scale = xs;
    a.a_rows = rs;
    a.b_scale = W.gu_s;
    a.out_bf16 = ab;
    a.out_ld = 2 * I;
    a.out_cols = 2 * I;
    rc = launch_chain("FP8 backward GEMM ab = X W_gu^T",
                      gemm8::k_gemm_promoted<2, gemm8::EPI_BF16_OUT>,
                      dim3(grid_of(mt_rows * a.n_tiles_n)), dim3(gemm8::NUM_THREADS), smem, st,
                      ta, tb, a);
    if (rc != MOE_OK) return rc;
  }
  // G2: dz' = dY W_down with the SwiGLU backward in the epilogue (W_down^T rows)
  {
    CUtensorMap ta, tb;
    rc = make_tmap(&ta, dhq, 1, d, rs, gemm8::BM);
    if (rc == MOE_OK) rc = make_tmap(&tb, W.down_t, 1, d, (uint64_t)E * I, gemm8::BN);
    if (rc != MOE_OK) return rc;
    gemm8::Args a = base_args(gtab, (I + gemm8::BN - 1) / gemm8::BN, d / 128, I);
    a.a_scale = dhs;
    a.a_rows = rs;
    a.b_scale = W.down_t_s;
    a.ab = ab;
    a.zg = zg;
    a.dab = dab;
    a.dgp = dgp;
    a.row_w = row_w;
    rc = launch_chain("FP8 backward GEMM dz = dY W_down",
                      gemm8::k_gemm_promoted<2, gemm8::EPI_SWIGLU_BWD>,
                      dim3(grid_of(mt_rows * a.n_tiles_n)), dim3(gemm8::NUM_THREADS), smem, st,
                      ta, tb, a);
    if (rc != MOE_OK) return rc;
  }
  // [da | db] rows to FP8
  rc = launch_chain("k_quant_rows", perm::k_quant_rows, dim3((rs + 7) / 8), dim3(256), 0, st,
                    static_cast<const __nv_bfloat16*>(dab), rs, 2 * I, dabq, dabs);
  if (rc != MOE_OK) return rc;
  // G3: du pieces = dAB W_gu (W_gu^T rows), scattered to the token-major slots
  {
    CUtensorMap ta, tb;
    rc = make_tmap(&ta, dabq, 1, 2 * I, rs, gemm8::BM);
    if (rc == MOE_OK) rc = make_tmap(&tb, W.gu_t, 1, 2 * I, (uint64_t)E * d, gemm8::BN);
    if (rc != MOE_OK) return rc;
    gemm8::Args a = base_args(gtab, d / gemm8::BN, 2 * I / 128, d);
    a.a_scale = dabs;
    a.a_rows = rs;
    a.b_scale = W.gu_t_s;
    a.y = dslots;
    a.d = d;
    a.pair_of = row_pair;
    a.topk_w = nullptr;
    rc = launch_chain("FP8 backward GEMM du = dAB W_gu",
                      gemm8::k_gemm_promoted<2, gemm8::EPI_SCATTER>,
                      dim3(grid_of(mt_rows * a.n_tiles_n)), dim3(gemm8::NUM_THREADS), smem, st,
                      ta, tb, a);
    if (rc != MOE_OK) return rc;
  }
  // gate-weight and affinity backward -> dl [T, N]
  {
    const route::Params p = route_params(s);
    const int n_it = I / 64;
    if (N <= 32) rc = launch_gate_bwd<1>(logits, p, idx, slot_of, offsets, poff, dgp, n_it, dl, st);
    else if (N <= 64) rc = launch_gate_bwd<2>(logits, p, idx, slot_of, offsets, poff, dgp, n_it, dl, st);
    else if (N <= 128) rc = launch_gate_bwd<4>(logits, p, idx, slot_of, offsets, poff, dgp, n_it, dl, st);
    else if (N <= 256) rc = launch_gate_bwd<8>(logits, p, idx, slot_of, offsets, poff, dgp, n_it, dl, st);
    else rc = launch_gate_bwd<16>(logits, p, idx, slot_of, offsets, poff, dgp, n_it, dl, st);
    if (rc != MOE_OK) return rc;
  }
  // the router's part of dx in bf16 (gating stays BF16), then dx
  auto nt = [](int64_t n) { return (n + gbwd::BN - 1) / gbwd::BN; };
  const Operand X{x, (uint64_t)d, (uint64_t)T};
  const Operand DL{dl, (uint64_t)N, (uint64_t)T}, WR{w_router, (uint64_t)d, (uint64_t)N};
  gbwd::Args ga;
  memset(&ga, 0, sizeof(ga));
  ga.n_probs = 1;
  ga.K = K;
  ga.Ks = Ks;
  ga.inter = I;
  ga.tab = tab_dxr;
  ga.c = dxr;
  ga.ldc = d;
  rc = launch_gemm_bwd<true, gbwd::EPI_BF16>("backward GEMM dx_router = dL W_r", DL, DL, WR, WR,
                                             ga, nt(d) * ((T + 127) / 128), st);
  if (rc != MOE_OK) return rc;
  rc = do_combine(D, dxr, dslots, dx, st);
  if (rc != MOE_OK) return rc;
  // weight-gradient operands: 128-row x 1-column tiles, transposed
  {
    const dim3 blk(256);
    rc = launch_chain("k_quant_cols dY", bwd8::k_quant_cols<true>, dim3(rs / 128, d / 64), blk, 0,
                      st, static_cast<const __nv_bfloat16*>(dh),
                      static_cast<const int32_t*>(row_tok), d, rs, ws + B.dhT,
                      reinterpret_cast<float*>(ws + B.dhTs));
    if (rc == MOE_OK)
      rc = launch_chain("k_quant_cols gz", bwd8::k_quant_cols<false>, dim3(rs / 128, I / 64), blk,
                        0, st, static_cast<const __nv_bfloat16*>(zg),
                        static_cast<const int32_t*>(nullptr), I, rs, ws + B.zgT,
                        reinterpret_cast<float*>(ws + B.zgTs));
    if (rc == MOE_OK)
      rc = launch_chain("k_quant_cols dAB", bwd8::k_quant_cols<false>,
                        dim3(rs / 128, 2 * I / 64), blk, 0, st,
                        static_cast<const __nv_bfloat16*>(dab),
                        static_cast<const int32_t*>(nullptr), 2 * I, rs, ws + B.dabT,
                        reinterpret_cast<float*>(ws + B.dabTs));
    if (rc == MOE_OK)
      rc = launch_chain("k_quant_cols X", bwd8::k_quant_cols<true>, dim3(rs / 128, d / 64), blk, 0,
                        st, static_cast<const __nv_bfloat16*>(x),
                        static_cast<const int32_t*>(row_tok), d, rs, ws + B.xT,
                        reinterpret_cast<float*>(ws + B.xTs));
    if (rc != MOE_OK) return rc;
  }
  // G4: dW_down = dY^T (g z) and G5: dW_gu = dAB^T X over each expert's rows,
  // bf16 out
  {
    CUtensorMap ta, tb;
    rc = make_tmap(&ta, ws + B.dhT, 1, rs, d, gemm8::BM);
    if (rc == MOE_OK) rc = make_tmap(&tb, ws + B.zgT, 1, rs, I, gemm8::WG_BN);
    if (rc != MOE_OK) return rc;
    gemm8::Args a = base_args(gtab_wd, (I + gemm8::WG_BN - 1) / gemm8::WG_BN, 0, 0);
    a.stages = wg_stages;
    a.idesc = umma_idesc(0, gemm8::BM, gemm8::WG_BN);
    a.kgroup = kgroup;
    a.a_scale = reinterpret_cast<const float*>(ws + B.dhTs);
    a.a_scale_ld = d;
    a.a_rows = d;
    a.b_scale = reinterpret_cast<const float*>(ws + B.zgTs);
    a.b_scale_ld = I;
    a.b_rows = I;
    a.out_bf16 = static_cast<__nv_bfloat16*>(dw_down);
    a.out_ld = I;
    a.out_cols = I;
    rc = launch_chain("FP8 backward GEMM dW_down = dY^T Z",
                      gemm8::k_gemm_promoted<2, gemm8::EPI_BF16_OUT, true>,
                      dim3(grid_of((int64_t)E * (d / 128) * a.n_tiles_n)),
                      dim3(gemm8::NUM_THREADS), wg_smem, st, ta, tb, a);
    if (rc != MOE_OK) return rc;
  }
  {
    CUtensorMap ta, tb;
    rc = make_tmap(&ta, ws + B.dabT, 1, rs, 2 * I, gemm8::BM);
    if (rc == MOE_OK) rc = make_tmap(&tb, ws + B.xT, 1, rs, d, gemm8::WG_BN);
    if (rc != MOE_OK) return rc;
    gemm8::Args a = base_args(gtab_wgu, d / gemm8::WG_BN, 0, 0);
    a.stages = wg_stages;
    a.idesc = umma_idesc(0, gemm8::BM, gemm8::WG_BN);
    a.kgroup = kgroup;
    a.a_scale = reinterpret_cast<const float*>(ws + B.dabTs);
    a.a_scale_ld = 2 * I;
    a.a_rows = 2 * I;
    a.b_scale = reinterpret_cast<const float*>(ws + B.xTs);
    a.b_scale_ld = d;
    a.b_rows = d;
    a.out_bf16 = static_cast<__nv_bfloat16*>(dw_gu);
    a.out_ld = d;
    a.out_cols = d;
    rc = launch_chain("FP8 backward GEMM dW_gu = dAB^T X",
                      gemm8::k_gemm_promoted<2, gemm8::EPI_BF16_OUT, true>,
                      dim3(grid_of((int64_t)E * (2 * I / 128) * a.n_tiles_n)),
                      dim3(gemm8::NUM_THREADS), wg_smem, st, ta, tb, a);
    if (rc != MOE_OK) return rc;
  }
  // G6b: dW_r = dl^T X (bf16 gating GEMM), bf16 out
  ga.tab = tab_dwr;
  ga.c = dw_router;
  ga.ldc = d;
  return launch_gemm_bwd_pair("backward GEMM dW_r = dL^T X (CTA pairs)", DL, DL, X, X, ga,
                              (uint64_t)N, 1, ((N + 255) / 256) * nt(d), true, st);
}

__global__ void k_selftest_wait(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing arrives on `bar`: the wait must give up after limit_ns.
    const uint64_t t0 = globaltimer_ns();
    bool done = false;
    while (!done) {
      if (mbar_try_wait(&bar, 0)) break;
      if (globaltimer_ns() - t0 > limit_ns) {
        set_status(MOE_ERR_TIMEOUT);
        done = true;
      }
    }
  }
  __syncthreads();
}


// ----------------------------------------------------------------------------- no-allocation permute
// Scratch of moe_permute_noalloc: the per-chunk histogram, in a fixed device
// array that every device loading this library holds until the process exits.
static __device__ __align__(256) int32_t g_noalloc_hist[MOE_NOALLOC_HIST_INTS];

// Device address of g_noalloc_hist, looked up once per device (host code
// cannot use the symbol itself: on the host it names a stand-in, not device
// memory).
int32_t* g_noalloc_ptr[kMaxDevices] = {};

moe_status noalloc_scratch(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_hist);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
    g_noalloc_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return MOE_OK;
}

}  // namespace

// ============================================================================= C ABI
extern "C" {

size_t moe_workspace_size(const moe_layer_desc* desc) {
  Dims D;
  if (fill_dims(desc, &D) != MOE_OK) return 0;
  return layout(D).total;
}

moe_status moe_route(const moe_layer_desc* desc, const void* x, const void* w_router,
                     const float* bias, int32_t* topk_idx, float* topk_w, int32_t* counts,
                     void* ws, size_t ws_bytes, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (bias && desc->gate != MOE_GATE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (!counts || !aligned16(counts)) return MOE_ERR_INVALID_ARG;
  if (D.T > 0) {
    if (!x || !w_router || !topk_idx || !topk_w || !aligned16(x) || !aligned16(w_router) ||
        !aligned16(topk_idx) || !aligned16(topk_w) || (bias && !aligned16(bias)))
      return MOE_ERR_INVALID_ARG;
  }
  const Layout L = layout(D);
  if (!ws || ws_bytes < L.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  int sms;
  if ((rc = device_setup(&sms)) != MOE_OK) return rc;
  return do_route(*desc, D, L, x, w_router, bias, topk_idx, topk_w, counts,
                  static_cast<uint8_t*>(ws), sms, stream);
}

moe_status moe_permute(const moe_layer_desc* desc, const void* x, const int32_t* topk_idx,
                       const int32_t* counts, int32_t* offsets, int32_t* perm_src,
                       int32_t* slot_of, void* x_perm, float* x_perm_scale, void* ws,
                       size_t ws_bytes, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (!offsets || !aligned16(offsets)) return MOE_ERR_INVALID_ARG;
  if (D.T > 0) {
    if (!x_perm && !x_perm_scale) {
      // maps only: x is not read
      if (!topk_idx || !counts || !perm_src || !slot_of || !aligned16(topk_idx) ||
          !aligned16(perm_src) || !aligned16(slot_of))
        return MOE_ERR_INVALID_ARG;
    } else {
      if (!x || !topk_idx || !counts || !perm_src || !slot_of || !x_perm || !aligned16(x) ||
          !aligned16(topk_idx) || !aligned16(perm_src) || !aligned16(slot_of) ||
          !aligned16(x_perm))
        return MOE_ERR_INVALID_ARG;
      if (D.fp8 != (x_perm_scale != nullptr)) return MOE_ERR_INVALID_ARG;
      if (x_perm_scale && !aligned16(x_perm_scale)) return MOE_ERR_INVALID_ARG;
    }
  }
  const Layout L = layout(D);
  if (!ws || ws_bytes < L.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  int sms;
  if ((rc = device_setup(&sms)) != MOE_OK) return rc;
  return do_permute(D, reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + L.hist), x,
                    topk_idx, counts, offsets, perm_src, slot_of, x_perm, x_perm_scale, stream);
}

moe_status moe_grouped_swiglu(const moe_layer_desc* desc, const void* x, const void* x_perm,
                              const float* x_perm_scale, const int32_t* offsets,
                              const int32_t* perm_src, const int32_t* slot_of,
                              const float* topk_w, const void* w_gu, const float* w_gu_scale,
                              const void* w_down, const float* w_down_scale, void* y_slots,
                              void* ws, size_t ws_bytes, cudaStream_t stream) {
  (void)perm_src;
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (D.T > 0) {
    if (!x_perm || !offsets || !slot_of || !topk_w || !w_gu || !w_down || !y_slots ||
        !aligned16(x_perm) || !aligned16(w_gu) || !aligned16(w_down) || !aligned16(y_slots))
      return MOE_ERR_INVALID_ARG;
    if (!D.fp8 && (!x || !aligned16(x))) return MOE_ERR_INVALID_ARG;
    if (D.fp8 && (!x_perm_scale || !w_gu_scale || !w_down_scale)) return MOE_ERR_INVALID_ARG;
  }
  const Layout L = layout(D);
  if (!ws || ws_bytes < L.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  int sms;
  if ((rc = device_setup(&sms)) != MOE_OK) return rc;
  return do_grouped(D, L, x, x_perm, x_perm_scale, offsets, slot_of, topk_w, w_gu, w_gu_scale,
                    w_down, w_down_scale, y_slots,
                    static_cast<uint8_t*>(ws), sms, stream);
}

moe_status moe_combine(const moe_layer_desc* desc, const void* x_residual, const void* y_slots,
                       void* h, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (D.T > 0 && (!x_residual || !y_slots || !h || !aligned16(x_residual) ||
                  !aligned16(y_slots) || !aligned16(h)))
    return MOE_ERR_INVALID_ARG;
  return do_combine(D, x_residual, y_slots, h, stream);
}

static moe_status forward_entry(const moe_layer_desc* desc, const void* x,
                                const void* x_residual, const void* w_router, const float* bias,
                                const void* w_gu, const float* w_gu_scale, const void* w_down,
                                const float* w_down_scale, void* h, int32_t* topk_idx,
                                int32_t* counts, void* ab_save, void* ws, size_t ws_bytes,
                                cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (bias && desc->gate != MOE_GATE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (D.T > 0) {
    if (!x || !w_router || !w_gu || !w_down || !h || !aligned16(x) || !aligned16(w_router) ||
        !aligned16(w_gu) || !aligned16(w_down) || !aligned16(h) || (bias && !aligned16(bias)) ||
        (x_residual && !aligned16(x_residual)) || (topk_idx && !aligned16(topk_idx)))
      return MOE_ERR_INVALID_ARG;
    if (D.fp8 && (!w_gu_scale || !w_down_scale)) return MOE_ERR_INVALID_ARG;
  }
  if (counts && !aligned16(counts)) return MOE_ERR_INVALID_ARG;
  const Layout L = layout(D);
  if (!ws || ws_bytes < L.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  int sms;
  if ((rc = device_setup(&sms)) != MOE_OK) return rc;
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  int32_t* idx = topk_idx ? topk_idx : reinterpret_cast<int32_t*>(w8 + L.topk_idx);
  float* tw = reinterpret_cast<float*>(w8 + L.topk_w);
  int32_t* cnt = counts ? counts : reinterpret_cast<int32_t*>(w8 + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(w8 + L.offsets);
  int32_t* perm_src = reinterpret_cast<int32_t*>(w8 + L.perm_src);
  int32_t* slot_of = reinterpret_cast<int32_t*>(w8 + L.slot_of);
  void* x_perm = w8 + L.x_perm;
  float* x_perm_scale = D.fp8 ? reinterpret_cast<float*>(w8 + L.x_perm_scale) : nullptr;
  void* y = w8 + L.y_slots;
  if ((rc = trace(0, stream)) != MOE_OK) return rc;
  if ((rc = do_route(*desc, D, L, x, w_router, bias, idx, tw, nullptr, w8, sms, stream)) !=
      MOE_OK)
    return rc;
  if ((rc = trace(1, stream)) != MOE_OK) return rc;
  // the permutation's histogram totals are the expert counts
  if ((rc = do_permute(D, reinterpret_cast<int32_t*>(w8 + L.hist), x, idx, nullptr, offsets,
                       perm_src, slot_of, x_perm, x_perm_scale, stream, cnt)) != MOE_OK)
    return rc;
  if ((rc = do_grouped(D, L, x, x_perm, x_perm_scale, offsets, slot_of, tw, w_gu, w_gu_scale,
                       w_down, w_down_scale, y, w8, sms, stream,
                       static_cast<__nv_bfloat16*>(ab_save))) != MOE_OK)
    return rc;
  rc = do_combine(D, x_residual ? x_residual : x, y, h, stream);
  if (rc == MOE_OK) rc = trace(5, stream);
  return rc;
}

moe_status moe_forward(const moe_layer_desc* desc, const void* x, const void* x_residual,
                       const void* w_router, const float* bias, const void* w_gu,
                       const float* w_gu_scale, const void* w_down, const float* w_down_scale,
                       void* h, int32_t* topk_idx, int32_t* counts, void* ws, size_t ws_bytes,
                       cudaStream_t stream) {
  return forward_entry(desc, x, x_residual, w_router, bias, w_gu, w_gu_scale, w_down,
                       w_down_scale, h, topk_idx, counts, nullptr, ws, ws_bytes, stream);
}

size_t moe_saved_ab_bytes(const moe_layer_desc* desc) {
  Dims D;
  if (fill_dims(desc, &D) != MOE_OK) return 0;
  if (D.act != MOE_DT_BF16 || D.w != MOE_DT_BF16) return 0;
  return (size_t)(D.R + D.Ks * D.T) * 2 * D.I * 2;
}

moe_status moe_forward_save(const moe_layer_desc* desc, const void* x, const void* x_residual,
                            const void* w_router, const float* bias, const void* w_gu,
                            const void* w_down, void* h, int32_t* topk_idx, int32_t* counts,
                            void* ab_saved, void* ws, size_t ws_bytes, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (D.act != MOE_DT_BF16 || D.w != MOE_DT_BF16) return MOE_ERR_UNSUPPORTED;
  if (D.T > 0 && (!ab_saved || !aligned16(ab_saved))) return MOE_ERR_INVALID_ARG;
  return forward_entry(desc, x, x_residual, w_router, bias, w_gu, nullptr, w_down, nullptr, h,
                       topk_idx, counts, ab_saved, ws, ws_bytes, stream);
}

moe_status moe_route_affinities(const moe_layer_desc* desc, const void* x, const void* w_router,
                                float* s_out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (D.T > 0 && (!x || !w_router || !s_out || !aligned16(x) || !aligned16(w_router) ||
                  !aligned16(s_out)))
    return MOE_ERR_INVALID_ARG;
  const Layout L = layout(D);
  if (!ws || ws_bytes < L.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  if (D.T == 0) return MOE_OK;
  int sms;
  if ((rc = device_setup(&sms)) != MOE_OK) return rc;
  const route::Params p = route_params(*desc);
  const int N = (int)D.N, blocks = (int)((D.T + 7) / 8);
  if (D.f32) {
    const float* xf = static_cast<const float*>(x);
    const float* wf = static_cast<const float*>(w_router);
    const int dd = (int)D.d;
    if (N <= 32) route::k_affinity_f32<1><<<blocks, 256, 0, stream>>>(xf, wf, dd, p, s_out);
    else if (N <= 64) route::k_affinity_f32<2><<<blocks, 256, 0, stream>>>(xf, wf, dd, p, s_out);
    else if (N <= 128) route::k_affinity_f32<4><<<blocks, 256, 0, stream>>>(xf, wf, dd, p, s_out);
    else if (N <= 256) route::k_affinity_f32<8><<<blocks, 256, 0, stream>>>(xf, wf, dd, p, s_out);
    else route::k_affinity_f32<16><<<blocks, 256, 0, stream>>>(xf, wf, dd, p, s_out);
    return launched("k_affinity_f32");
  }
  float* logits = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.logits);
  if ((rc = launch_router(D, x, w_router, logits, nullptr, sms, stream)) != MOE_OK) return rc;
  if (N <= 32) route::k_affinity<1><<<blocks, 256, 0, stream>>>(logits, p, s_out);
  else if (N <= 64) route::k_affinity<2><<<blocks, 256, 0, stream>>>(logits, p, s_out);
  else if (N <= 128) route::k_affinity<4><<<blocks, 256, 0, stream>>>(logits, p, s_out);
  else if (N <= 256) route::k_affinity<8><<<blocks, 256, 0, stream>>>(logits, p, s_out);
  else route::k_affinity<16><<<blocks, 256, 0, stream>>>(logits, p, s_out);
  return launched("k_affinity");
}

moe_status moe_balance_stats(const moe_layer_desc* desc, const float* s, const int32_t* topk_idx,
                             int32_t seq_len, float* f_out, float* p_out, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (D.T == 0) return MOE_OK;
  if (seq_len <= 0 || D.T % seq_len) return MOE_ERR_INVALID_ARG;
  if (!s || !topk_idx || !f_out || !p_out || !aligned16(s) || !aligned16(topk_idx))
    return MOE_ERR_INVALID_ARG;
  const dim3 grid((unsigned)(D.T / seq_len), (unsigned)((D.N + 31) / 32));
  route::k_balance_stats<<<grid, 256, 0, stream>>>(s, topk_idx, (int)D.T, (int)D.N, (int)D.K,
                                                   seq_len, f_out, p_out);
  return launched("k_balance_stats");
}

moe_status moe_bias_update(const moe_layer_desc* desc, const int32_t* counts, float* bias,
                           float gamma, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (!counts || !bias || !std::isfinite(gamma) || gamma < 0.f) return MOE_ERR_INVALID_ARG;
  route::k_bias_update<<<1, 512, 0, stream>>>(counts, bias, (int)D.N, (long long)D.T * D.K, gamma);
  return launched("k_bias_update");
}

moe_status moe_quantize_fp8_blockwise(const void* w_bf16, int32_t rows, int32_t cols,
                                      int32_t batch, void* w_e4m3, float* scale,
                                      cudaStream_t stream) {
  if (rows <= 0 || cols <= 0 || batch <= 0 || rows % 128 || cols % 128) return MOE_ERR_INVALID_ARG;
  if (!w_bf16 || !w_e4m3 || !scale || !aligned16(w_bf16) || !aligned16(w_e4m3))
    return MOE_ERR_INVALID_ARG;
  const int64_t blocks = (int64_t)batch * (rows / 128) * (cols / 128);
  if (blocks >= ((int64_t)1 << 31)) return MOE_ERR_INVALID_ARG;
  perm::k_quant_w<false><<<(unsigned)blocks, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(w_bf16), rows, cols, static_cast<uint8_t*>(w_e4m3), scale);
  return launched("k_quant_w");
}

moe_status moe_quantize_fp8_blockwise_t(const void* w_bf16, int32_t rows, int32_t cols,
                                        int32_t batch, void* w_e4m3_t, float* scale_t,
                                        cudaStream_t stream) {
  if (rows <= 0 || cols <= 0 || batch <= 0 || rows % 128 || cols % 128) return MOE_ERR_INVALID_ARG;
  if (!w_bf16 || !w_e4m3_t || !scale_t || !aligned16(w_bf16) || !aligned16(w_e4m3_t))
    return MOE_ERR_INVALID_ARG;
  const int64_t blocks = (int64_t)batch * (rows / 128) * (cols / 128);
  if (blocks >= ((int64_t)1 << 31)) return MOE_ERR_INVALID_ARG;
  perm::k_quant_w<true><<<(unsigned)blocks, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(w_bf16), rows, cols, static_cast<uint8_t*>(w_e4m3_t),
      scale_t);
  return launched("k_quant_w (transposed)");
}

const char* moe_status_string(moe_status status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE_CHECK: return "device consistency check failed";
  }
  return "unknown status";
}

moe_status moe_last_device_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  return static_cast<moe_status>(v);
}

moe_status moe_trace_events(cudaEvent_t* events, int32_t n) {
  if (events && n != 6) return MOE_ERR_INVALID_ARG;
  t_events = events;
  return MOE_OK;
}

const char* moe_last_error_message(void) { return t_errmsg; }

int32_t moe_forward_launch_count(const moe_layer_desc* desc) {
  Dims D;
  if (fill_dims(desc, &D) != MOE_OK) return 0;
  if (D.T == 0) return 2;
  // route (router GEMM + top-K; fp32: one kernel) + permute (4) + grouped (3)
  // + combine (1)
  return (D.f32 ? 1 : 2) + 4 + 3 + 1;
}

moe_status moe_selftest_bounded_wait(uint32_t limit_us, cudaStream_t stream) {
  if (limit_us < 1 || limit_us > 1000000) return MOE_ERR_INVALID_ARG;
  k_selftest_wait<<<1, 32, 0, stream>>>((uint64_t)limit_us * 1000ull);
  return launched("k_selftest_wait");
}

moe_status moe_permute_noalloc(const moe_layer_desc* desc, const void* x,
                               const int32_t* topk_idx, const int32_t* counts, int32_t* offsets,
                               int32_t* perm_src, int32_t* slot_of, void* x_perm,
                               float* x_perm_scale, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (!offsets || !aligned16(offsets)) return MOE_ERR_INVALID_ARG;
  if (D.T > 0) {
    if (!x || !topk_idx || !counts || !perm_src || !slot_of || !x_perm || !aligned16(x) ||
        !aligned16(topk_idx) || !aligned16(perm_src) || !aligned16(slot_of) ||
        !aligned16(x_perm))
      return MOE_ERR_INVALID_ARG;
    if (D.fp8 != (x_perm_scale != nullptr)) return MOE_ERR_INVALID_ARG;
    if (x_perm_scale && !aligned16(x_perm_scale)) return MOE_ERR_INVALID_ARG;
  }
  const int64_t need = (int64_t)D.n_chunks * D.N;
  if (need > MOE_NOALLOC_HIST_INTS) {
    snprintf(t_errmsg, sizeof(t_errmsg),
             "moe_permute_noalloc: ceil(T/128)*N = %lld histogram entries exceed the fixed "
             "scratch of %d; use moe_permute with a workspace",
             (long long)need, (int)MOE_NOALLOC_HIST_INTS);
    return MOE_ERR_UNSUPPORTED;
  }
  int sms;
  if ((rc = device_setup(&sms)) != MOE_OK) return rc;
  int32_t* hist = nullptr;
  if ((rc = noalloc_scratch(&hist)) != MOE_OK) return rc;
  // The same launch chain as moe_permute.  Every histogram entry the scan
  // reads is written first by k_hist, so the previous call's contents never
  // leak into this one.
  return do_permute(D, hist, x, topk_idx, counts, offsets, perm_src, slot_of, x_perm,
                    x_perm_scale, stream);
}

size_t moe_backward_workspace_size(const moe_layer_desc* desc) {
  Dims D;
  if (fill_dims(desc, &D) != MOE_OK) return 0;
  if (D.act != MOE_DT_BF16 || D.w != MOE_DT_BF16) return 0;
  const Layout L = layout(D);
  return bwd_layout(D, L).total;
}

static moe_status backward_entry(const moe_layer_desc* desc, const void* x,
                                 const void* w_router, const float* bias, const void* w_gu,
                                 const void* w_down, const void* dh, void* dx, void* dw_router,
                                 void* dw_gu, void* dw_down, bool bf16_grads,
                                 const void* ab_saved, void* ws, size_t ws_bytes,
                                 cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (D.act != MOE_DT_BF16 || D.w != MOE_DT_BF16) return MOE_ERR_UNSUPPORTED;
  if (bias && desc->gate != MOE_GATE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (D.E > 1024) return MOE_ERR_UNSUPPORTED;
  if (D.T > 0) {
    if (!x || !w_router || !w_gu || !w_down || !dh || !dx || !dw_router || !dw_gu || !dw_down ||
        !aligned16(x) || !aligned16(w_router) || !aligned16(w_gu) || !aligned16(w_down) ||
        !aligned16(dh) || !aligned16(dx) || !aligned16(dw_router) || !aligned16(dw_gu) ||
        !aligned16(dw_down) || (bias && !aligned16(bias)) || (ab_saved && !aligned16(ab_saved)))
      return MOE_ERR_INVALID_ARG;
    if ((D.N * 2) % 16) return MOE_ERR_UNSUPPORTED;   // rows of dl must be 16-byte aligned
  }
  const Layout L = layout(D);
  const BwdLayout B = bwd_layout(D, L);
  if (!ws || ws_bytes < B.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  if (B.rows >= ((int64_t)1 << 31)) return MOE_ERR_INVALID_ARG;
  if (D.T == 0) return MOE_OK;
  int sms;
  if ((rc = device_setup(&sms)) != MOE_OK) return rc;
  return do_backward(*desc, D, L, B, x, w_router, bias, w_gu, w_down, dh, dx, dw_router, dw_gu,
                     dw_down, bf16_grads, ab_saved, static_cast<uint8_t*>(ws), sms, stream);
}

moe_status moe_backward(const moe_layer_desc* desc, const void* x, const void* w_router,
                        const float* bias, const void* w_gu, const void* w_down, const void* dh,
                        void* dx, float* dw_router, float* dw_gu, float* dw_down, void* ws,
                        size_t ws_bytes, cudaStream_t stream) {
  return backward_entry(desc, x, w_router, bias, w_gu, w_down, dh, dx, dw_router, dw_gu, dw_down,
                        false, nullptr, ws, ws_bytes, stream);
}

moe_status moe_backward_bf16_grads(const moe_layer_desc* desc, const void* x,
                                   const void* w_router, const float* bias, const void* w_gu,
                                   const void* w_down, const void* dh, void* dx, void* dw_router,
                                   void* dw_gu, void* dw_down, void* ws, size_t ws_bytes,
                                   cudaStream_t stream) {
  return backward_entry(desc, x, w_router, bias, w_gu, w_down, dh, dx, dw_router, dw_gu, dw_down,
                        true, nullptr, ws, ws_bytes, stream);
}

moe_status moe_backward_saved(const moe_layer_desc* desc, const void* x, const void* w_router,
                              const float* bias, const void* w_gu, const void* w_down,
                              const void* dh, const void* ab_saved, void* dx, void* dw_router,
                              void* dw_gu, void* dw_down, int32_t bf16_grads, void* ws,
                              size_t ws_bytes, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (D.T > 0 && !ab_saved) return MOE_ERR_INVALID_ARG;
  return backward_entry(desc, x, w_router, bias, w_gu, w_down, dh, dx, dw_router, dw_gu, dw_down,
                        bf16_grads != 0, ab_saved, ws, ws_bytes, stream);
}

size_t moe_backward_fp8_workspace_size(const moe_layer_desc* desc) {
  Dims D;
  if (fill_dims(desc, &D) != MOE_OK || !D.fp8) return 0;
  return bwd8_layout(D, layout(D)).total;
}

moe_status moe_backward_fp8(const moe_layer_desc* desc, const void* x, const void* w_router,
                            const float* bias, const void* w_gu, const float* w_gu_scale,
                            const void* w_gu_t, const float* w_gu_t_scale, const void* w_down_t,
                            const float* w_down_t_scale, const void* dh, void* dx,
                            void* dw_router, void* dw_gu, void* dw_down, void* ws,
                            size_t ws_bytes, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (!D.fp8) return MOE_ERR_UNSUPPORTED;
  if (bias && desc->gate != MOE_GATE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (D.E > 1024 || D.K + D.Ks > 32 || D.d % 256 || (D.N * 2) % 16) return MOE_ERR_UNSUPPORTED;
  if (D.T > 0) {
    const void* need[] = {x, w_router, w_gu, w_gu_t, w_down_t, dh, dx, dw_router, dw_gu, dw_down};
    for (const void* p : need)
      if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
    const float* scales[] = {w_gu_scale, w_gu_t_scale, w_down_t_scale};
    for (const float* p : scales)
      if (!p || ((uintptr_t)p & 3u)) return MOE_ERR_INVALID_ARG;
    if (bias && !aligned16(bias)) return MOE_ERR_INVALID_ARG;
  }
  const Layout L = layout(D);
  const Bwd8Layout B = bwd8_layout(D, L);
  if (!ws || ws_bytes < B.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  if (B.rs >= ((int64_t)1 << 31) / 2) return MOE_ERR_INVALID_ARG;
  if (D.T == 0) return MOE_OK;
  int sms;
  if ((rc = device_setup(&sms)) != MOE_OK) return rc;
  const Fp8Weights W{w_gu, w_gu_t, w_down_t, w_gu_scale, w_gu_t_scale, w_down_t_scale};
  return do_backward_fp8(*desc, D, L, B, x, w_router, bias, W, dh, dx, dw_router, dw_gu, dw_down,
                         static_cast<uint8_t*>(ws), sms, stream);
}

int32_t moe_backward_fp8_launch_count(const moe_layer_desc* desc) {
  Dims D;
  if (fill_dims(desc, &D) != MOE_OK || !D.fp8) return 0;
  if (D.T == 0) return 0;
  // route (2) + hist, scan, slots (3) + prep, gather, pads (3) + ab, dz, the dAB
  // quantisation, du (4) + gate backward, dx_router, combine (3) + four
  // column quantisations + dW_down, dW_gu, dW_r (7)
  return 2 + 3 + 3 + 4 + 3 + 7;
}

int32_t moe_backward_launch_count(const moe_layer_desc* desc) {
  Dims D;
  if (fill_dims(desc, &D) != MOE_OK) return 0;
  if (D.T == 0) return 0;
  // route (2) + hist, scan, slots (3) + prep, gather, zero pads (3) + six GEMMs on the
  // rows and experts + gate backward + combine + the router-weight GEMM
  return 2 + 3 + 3 + 6 + 1 + 1 + 1;
}

size_t moe_expert_ffn_workspace_size(const moe_layer_desc* desc, int32_t n_groups,
                                     int32_t n_rows_out) {
  Dims D;
  if (fill_dims(desc, &D) != MOE_OK || n_groups < 1 || n_rows_out < 0) return 0;
  return ffn_layout(D, n_groups, n_rows_out).total;
}

moe_status moe_expert_ffn(const moe_layer_desc* desc, int32_t n_experts, int32_t n_groups,
                          const int32_t* groups, int32_t n_rows_in, int32_t n_rows_out,
                          const void* x_rows, const float* row_w, const void* w_gu,
                          const void* w_down, void* y_rows, void* ws, size_t ws_bytes,
                          cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (D.fp8) return MOE_ERR_UNSUPPORTED;
  if (n_experts < 1 || n_groups < 1 || n_groups > 1024 || n_rows_in < 0 || n_rows_out < 0)
    return MOE_ERR_INVALID_ARG;
  if (!groups || !aligned16(groups) || !w_gu || !w_down || !aligned16(w_gu) ||
      !aligned16(w_down))
    return MOE_ERR_INVALID_ARG;
  if (n_rows_out > 0 && (!y_rows || !aligned16(y_rows))) return MOE_ERR_INVALID_ARG;
  if (n_rows_in > 0 && (!x_rows || !aligned16(x_rows))) return MOE_ERR_INVALID_ARG;
  const FfnLayout F = ffn_layout(D, n_groups, n_rows_out);
  if (!ws || ws_bytes < F.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  if (n_rows_out == 0 || n_rows_in == 0) return MOE_OK;
  int sms;
  if ((rc = device_setup(&sms)) != MOE_OK) return rc;
  return do_expert_ffn(D, n_experts, n_groups, groups, n_rows_in, n_rows_out, x_rows, row_w, w_gu,
                       w_down, y_rows, nullptr, static_cast<uint8_t*>(ws), sms, stream);
}

moe_status moe_expert_ffn_fp8(const moe_layer_desc* desc, int32_t n_experts, int32_t n_groups,
                              const int32_t* groups, int32_t n_rows_in, int32_t n_rows_out,
                              const void* x_rows, const float* x_rows_scale, const float* row_w,
                              const void* w_gu, const float* w_gu_scale, const void* w_down,
                              const float* w_down_scale, void* y_rows, const uint64_t* group_out,
                              void* ws, size_t ws_bytes, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (!D.fp8) return MOE_ERR_INVALID_ARG;
  if (n_experts < 1 || n_groups < 1 || n_groups > 1024 || n_rows_in < 0 || n_rows_out < 0)
    return MOE_ERR_INVALID_ARG;
  if (!groups || !aligned16(groups) || !w_gu || !w_down || !aligned16(w_gu) ||
      !aligned16(w_down) || !w_gu_scale || !w_down_scale)
    return MOE_ERR_INVALID_ARG;
  if ((y_rows == nullptr) == (group_out == nullptr)) return MOE_ERR_INVALID_ARG;
  if (y_rows && n_rows_out > 0 && !aligned16(y_rows)) return MOE_ERR_INVALID_ARG;
  if (group_out && (reinterpret_cast<uintptr_t>(group_out) & 7u)) return MOE_ERR_INVALID_ARG;
  if (n_rows_in > 0 && (!x_rows || !aligned16(x_rows) || !x_rows_scale))
    return MOE_ERR_INVALID_ARG;
  const FfnLayout F = ffn_layout(D, n_groups, n_rows_out);
  if (!ws || ws_bytes < F.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  if (n_rows_out == 0 || n_rows_in == 0) return MOE_OK;
  int sms;
  if ((rc = device_setup(&sms)) != MOE_OK) return rc;
  return do_expert_ffn_fp8(D, n_experts, n_groups, groups, n_rows_in, n_rows_out, x_rows,
                           x_rows_scale, row_w, w_gu, w_gu_scale, w_down, w_down_scale, y_rows,
                           group_out, static_cast<uint8_t*>(ws), sms, stream);
}

moe_status moe_expert_ffn_to(const moe_layer_desc* desc, int32_t n_experts, int32_t n_groups,
                             const int32_t* groups, int32_t n_rows_in, int32_t n_rows_out,
                             const void* x_rows, const float* row_w, const void* w_gu,
                             const void* w_down, const uint64_t* group_out, void* ws,
                             size_t ws_bytes, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (D.fp8) return MOE_ERR_UNSUPPORTED;
  if (n_experts < 1 || n_groups < 1 || n_groups > 1024 || n_rows_in < 0 || n_rows_out < 0)
    return MOE_ERR_INVALID_ARG;
  if (!groups || !aligned16(groups) || !w_gu || !w_down || !aligned16(w_gu) ||
      !aligned16(w_down) || !group_out || (reinterpret_cast<uintptr_t>(group_out) & 7u))
    return MOE_ERR_INVALID_ARG;
  if (n_rows_in > 0 && (!x_rows || !aligned16(x_rows))) return MOE_ERR_INVALID_ARG;
  const FfnLayout F = ffn_layout(D, n_groups, n_rows_out);
  if (!ws || ws_bytes < F.total || !aligned16(ws)) return MOE_ERR_WORKSPACE;
  if (n_rows_out == 0 || n_rows_in == 0) return MOE_OK;
  int sms;
  if ((rc = device_setup(&sms)) != MOE_OK) return rc;
  return do_expert_ffn(D, n_experts, n_groups, groups, n_rows_in, n_rows_out, x_rows, row_w, w_gu,
                       w_down, nullptr, group_out, static_cast<uint8_t*>(ws), sms, stream);
}

moe_status moe_combine_rows(const moe_layer_desc* desc, const void* x_residual,
                            const void* y_shared, const void* y_rows, const int32_t* row_of,
                            int32_t n_rows, void* h, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (n_rows < 0) return MOE_ERR_INVALID_ARG;
  if (D.T == 0) return MOE_OK;
  if (!x_residual || !h || !row_of || !aligned16(x_residual) || !aligned16(h) ||
      (D.Ks > 0 && (!y_shared || !aligned16(y_shared))) ||
      (n_rows > 0 && (!y_rows || !aligned16(y_rows))))
    return MOE_ERR_INVALID_ARG;
  const int vec = D.f32 ? 4 : 8;
  const int64_t threads = D.T * (D.d / vec);
  const int blocks = (int)((threads + 255) / 256);
  if (D.f32)
    return launch_chain("k_combine_rows", perm::k_combine_rows<false>, dim3(blocks), dim3(256), 0,
                        stream, x_residual, y_shared, y_rows, row_of, (int)n_rows, h, (int)D.T,
                        (int)D.d, (int)D.K, (int)D.Ks);
  return launch_chain("k_combine_rows", perm::k_combine_rows<true>, dim3(blocks), dim3(256), 0,
                      stream, x_residual, y_shared, y_rows, row_of, (int)n_rows, h, (int)D.T,
                      (int)D.d, (int)D.K, (int)D.Ks);
}

moe_status moe_dispatch_rows(const moe_layer_desc* desc, const void* x, const float* topk_w,
                             const int32_t* row_of, int32_t n_rows, void* x_rows, float* w_rows,
                             cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (D.fp8) return MOE_ERR_UNSUPPORTED;
  if (n_rows < 0) return MOE_ERR_INVALID_ARG;
  if (D.T == 0) return MOE_OK;
  if (!x || !row_of || !x_rows || !aligned16(x) || !aligned16(x_rows) || (w_rows && !topk_w))
    return MOE_ERR_INVALID_ARG;
  perm::PeerDest none;
  memset(&none, 0, sizeof(none));
  return launch_chain("k_dispatch_rows", perm::k_dispatch_rows<false, false>,
                      dim3((unsigned)((D.T + 7) / 8)), dim3(256), 0, stream,
                      static_cast<const uint8_t*>(x), (int)D.T, (int)D.K, (int)(D.d * D.x_esz),
                      topk_w, row_of, (int)n_rows, static_cast<uint8_t*>(x_rows), w_rows,
                      static_cast<float*>(nullptr), none);
}

moe_status moe_dispatch_rows_fp8(const moe_layer_desc* desc, const void* x, const float* topk_w,
                                 const int32_t* row_of, int32_t n_rows, void* x_rows,
                                 float* x_rows_scale, float* w_rows, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (!D.fp8) return MOE_ERR_INVALID_ARG;
  if (n_rows < 0) return MOE_ERR_INVALID_ARG;
  if (D.T == 0) return MOE_OK;
  if (!x || !row_of || !x_rows || !x_rows_scale || !aligned16(x) || !aligned16(x_rows) ||
      (w_rows && !topk_w))
    return MOE_ERR_INVALID_ARG;
  perm::PeerDest none;
  memset(&none, 0, sizeof(none));
  return launch_chain("k_dispatch_rows", perm::k_dispatch_rows<false, true>,
                      dim3((unsigned)((D.T + 7) / 8)), dim3(256), 0, stream,
                      static_cast<const uint8_t*>(x), (int)D.T, (int)D.K, (int)D.d, topk_w,
                      row_of, (int)n_rows, static_cast<uint8_t*>(x_rows), w_rows, x_rows_scale,
                      none);
}

moe_status moe_quantize_rows_fp8(const moe_layer_desc* desc, const void* x, int32_t n_rows,
                                 void* codes, float* scales, cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (!D.fp8 || n_rows < 0) return MOE_ERR_INVALID_ARG;
  if (n_rows == 0) return MOE_OK;
  if (!x || !codes || !scales || !aligned16(x) || !aligned16(codes)) return MOE_ERR_INVALID_ARG;
  return launch_chain("k_quant_rows", perm::k_quant_rows, dim3((unsigned)((n_rows + 7) / 8)),
                      dim3(256), 0, stream, static_cast<const __nv_bfloat16*>(x), (int)n_rows,
                      (int)D.d, static_cast<uint8_t*>(codes), scales);
}

moe_status moe_dispatch_rows_to(const moe_layer_desc* desc, const void* x, const float* topk_w,
                                const int32_t* row_of, int32_t n_rows, const moe_peer_rows* dst,
                                cudaStream_t stream) {
  Dims D;
  moe_status rc = fill_dims(desc, &D);
  if (rc != MOE_OK) return rc;
  if (n_rows < 0 || !dst || dst->n_ranks < 1 || dst->n_ranks > MOE_MAX_PEERS)
    return MOE_ERR_INVALID_ARG;
  if (D.T == 0) return MOE_OK;
  if (!x || !row_of || !aligned16(x) || !topk_w) return MOE_ERR_INVALID_ARG;
  perm::PeerDest P;
  memset(&P, 0, sizeof(P));
  P.n = dst->n_ranks;
  if (dst->start[0] != 0 || dst->start[P.n] != n_rows) return MOE_ERR_INVALID_ARG;
  for (int q = 0; q < P.n; ++q) {
    if (dst->start[q + 1] < dst->start[q] || dst->base[q] < 0) return MOE_ERR_INVALID_ARG;
    if (dst->start[q + 1] > dst->start[q] &&
        (!dst->x[q] || !aligned16(dst->x[q]) || (D.fp8 && !dst->scale[q])))
      return MOE_ERR_INVALID_ARG;
    P.x[q] = static_cast<uint8_t*>(dst->x[q]);
    P.w[q] = dst->w[q];
    P.s[q] = dst->scale[q];
    P.start[q] = dst->start[q];
    P.base[q] = dst->base[q];
  }
  P.start[P.n] = dst->start[P.n];
  if (D.fp8)
    return launch_chain("k_dispatch_rows", perm::k_dispatch_rows<true, true>,
                        dim3((unsigned)((D.T + 7) / 8)), dim3(256), 0, stream,
                        static_cast<const uint8_t*>(x), (int)D.T, (int)D.K, (int)D.d, topk_w,
                        row_of, (int)n_rows, static_cast<uint8_t*>(nullptr),
                        static_cast<float*>(nullptr), static_cast<float*>(nullptr), P);
  return launch_chain("k_dispatch_rows", perm::k_dispatch_rows<true, false>,
                      dim3((unsigned)((D.T + 7) / 8)), dim3(256), 0, stream,
                      static_cast<const uint8_t*>(x), (int)D.T, (int)D.K, (int)(D.d * D.x_esz),
                      topk_w, row_of, (int)n_rows, static_cast<uint8_t*>(nullptr),
                      static_cast<float*>(nullptr), static_cast<float*>(nullptr), P);
}

moe_status moe_ipc_get_handle(const void* dev_ptr, void* handle, uint64_t* offset) {
  if (!dev_ptr || !handle || !offset) return MOE_ERR_INVALID_ARG;
  static_assert(sizeof(cudaIpcMemHandle_t) == MOE_IPC_HANDLE_BYTES, "IPC handle size");
  // the handle names the whole allocation (a caching allocator hands out
  // pieces of larger ones): find the allocation's base for the offset
  typedef CUresult (*RangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);
  static RangeFn range = nullptr;
  if (!range) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn) {
      snprintf(t_errmsg, sizeof(t_errmsg), "cuMemGetAddressRange entry point not found");
      return MOE_ERR_CUDA;
    }
    range = reinterpret_cast<RangeFn>(fn);
  }
  CUdeviceptr base = 0;
  size_t size = 0;
  const CUresult r = range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr));
  if (r != CUDA_SUCCESS) {
    snprintf(t_errmsg, sizeof(t_errmsg), "cuMemGetAddressRange: CUresult %d", (int)r);
    return MOE_ERR_CUDA;
  }
  cudaIpcMemHandle_t h;
  const cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcGetMemHandle");
  memcpy(handle, &h, sizeof(h));
  *offset = (uint64_t)(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
  return MOE_OK;
}

moe_status moe_ipc_open(const void* handle, void** dev_ptr) {
  if (!handle || !dev_ptr) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof(h));
  const cudaError_t e = cudaIpcOpenMemHandle(dev_ptr, h, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcOpenMemHandle");
  return MOE_OK;
}

moe_status moe_ipc_close(void* dev_ptr) {
  if (!dev_ptr) return MOE_ERR_INVALID_ARG;
  const cudaError_t e = cudaIpcCloseMemHandle(dev_ptr);
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcCloseMemHandle");
  return MOE_OK;
}

}  // extern "C"
