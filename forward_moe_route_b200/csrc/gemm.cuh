// Pieces shared by the grouped GEMMs: the device-built group table that maps
// tiles to experts and rows, the tile-to-group search, and epilogue helpers.
//
// The group table is built on the device from the permutation offsets, so
// nothing returns to the host between routing and the GEMMs.
#pragma once

#include "common.cuh"

namespace moe {
namespace gemm {

constexpr int BM = 128;            // rows of a group-table m-tile (the promoted GEMMs' UMMA M)
constexpr int KB = 128;            // bytes of K per stage = one 128-byte swizzle row

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

}  // namespace gemm
}  // namespace moe
