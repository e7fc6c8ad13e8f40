// Host and device fill routines of the counter-based synthetic generator.
//
// Element k of a fill is the generator's element (offset + k) of the tensor
// stream (seed, tensor_id), so a block of a tensor (one expert, one row
// range) is produced by the same call with the block's flat offset.  Host and
// device produce bit-identical values (see synth_core.h).
#include <cuda_runtime.h>
#include <stdint.h>
#include <thread>
#include <vector>

#include "synth_core.h"

namespace {

template <class F>
void host_parallel(uint64_t n, int nthreads, F&& body) {
  if (nthreads < 1) nthreads = 1;
  if (n < (1u << 16)) nthreads = 1;
  if (nthreads == 1) {
    body(0, n);
    return;
  }
  std::vector<std::thread> pool;
  uint64_t chunk = (n + nthreads - 1) / nthreads;
  for (int i = 0; i < nthreads; ++i) {
    uint64_t b = (uint64_t)i * chunk, e = b + chunk < n ? b + chunk : n;
    if (b >= e) break;
    pool.emplace_back([=, &body] { body(b, e); });
  }
  for (auto& t : pool) t.join();
}

__global__ void k_normal_f32(float* out, uint64_t n, uint64_t key, uint64_t off, float scale) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = syn_normal_f32(key, off + i, scale);
}

__global__ void k_normal_bf16(uint16_t* out, uint64_t n, uint64_t key, uint64_t off, float scale) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = syn_f32_to_bf16_bits(syn_normal_f32(key, off + i, scale));
}

__global__ void k_uniform_f32(float* out, uint64_t n, uint64_t key, uint64_t off, float lo, float hi) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = syn_uniform_f32(key, off + i, lo, hi);
}

unsigned grid_for(uint64_t n) {
  uint64_t b = (n + 255) / 256;
  return (unsigned)(b < 148u * 64u ? (b ? b : 1) : 148u * 64u);
}

}  // namespace

extern "C" {

uint64_t syn_key_of(uint64_t seed, uint64_t tensor_id) { return syn_key(seed, tensor_id); }

int syn_host_normal_f32(float* out, uint64_t n, uint64_t seed, uint64_t tensor_id, uint64_t offset,
                        float scale, int nthreads) {
  if (!out && n) return 1;
  uint64_t key = syn_key(seed, tensor_id);
  host_parallel(n, nthreads, [&](uint64_t b, uint64_t e) {
    for (uint64_t i = b; i < e; ++i) out[i] = syn_normal_f32(key, offset + i, scale);
  });
  return 0;
}

int syn_host_normal_bf16(uint16_t* out, uint64_t n, uint64_t seed, uint64_t tensor_id,
                         uint64_t offset, float scale, int nthreads) {
  if (!out && n) return 1;
  uint64_t key = syn_key(seed, tensor_id);
  host_parallel(n, nthreads, [&](uint64_t b, uint64_t e) {
    for (uint64_t i = b; i < e; ++i)
      out[i] = syn_f32_to_bf16_bits(syn_normal_f32(key, offset + i, scale));
  });
  return 0;
}

int syn_host_uniform_f32(float* out, uint64_t n, uint64_t seed, uint64_t tensor_id,
                         uint64_t offset, float lo, float hi, int nthreads) {
  if (!out && n) return 1;
  uint64_t key = syn_key(seed, tensor_id);
  host_parallel(n, nthreads, [&](uint64_t b, uint64_t e) {
    for (uint64_t i = b; i < e; ++i) out[i] = syn_uniform_f32(key, offset + i, lo, hi);
  });
  return 0;
}

// Device fills: asynchronous on `stream`; return the cudaError_t of the launch.
int syn_dev_normal_f32(float* out, uint64_t n, uint64_t seed, uint64_t tensor_id, uint64_t offset,
                       float scale, void* stream) {
  if (!n) return 0;
  k_normal_f32<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(out, n, syn_key(seed, tensor_id),
                                                              offset, scale);
  return (int)cudaGetLastError();
}

int syn_dev_normal_bf16(uint16_t* out, uint64_t n, uint64_t seed, uint64_t tensor_id,
                        uint64_t offset, float scale, void* stream) {
  if (!n) return 0;
  k_normal_bf16<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(out, n, syn_key(seed, tensor_id),
                                                               offset, scale);
  return (int)cudaGetLastError();
}

int syn_dev_uniform_f32(float* out, uint64_t n, uint64_t seed, uint64_t tensor_id,
                        uint64_t offset, float lo, float hi, void* stream) {
  if (!n) return 0;
  k_uniform_f32<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(out, n, syn_key(seed, tensor_id),
                                                               offset, lo, hi);
  return (int)cudaGetLastError();
}

}  // extern "C"
