// Shared device/host helpers of libvdn (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/vdn.h"

namespace vdn {

// Device status word bits (stored in the first 4 bytes of the workspace).
enum : int { kDevTimeout = 1, kDevRange = 2 };

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Query-token groups of one (b, h).  Group 0: anchor frame 0; group 1: anchor
// frame T-1 (T >= 2); groups 2..: the non-anchor frames of chunk c.  Every
// query in a group sees the same key segments (at most three contiguous token
// ranges: anchor frame 0, the window, anchor frame T-1).
struct QGroup {
  int row0, nrows;  // token range of the group
  int nseg;
  int seg0[3], seg1[3];  // key token ranges [seg0, seg1)
};

struct Geo {
  int T, N, C, R;  // frames, tokens/frame, chunk, window radius
  __host__ __device__ int n_chunks() const { return (T + C - 1) / C; }
  __host__ __device__ int n_groups() const { return T >= 2 ? 2 + n_chunks() : 1; }

  __host__ __device__ QGroup group(int g) const {
    QGroup q;
    const int L = T * N;
    if (g == 0 || g == 1) {
      const int f = (g == 0) ? 0 : T - 1;
      q.row0 = f * N;
      q.nrows = N;
      q.nseg = 1;
      q.seg0[0] = 0;
      q.seg1[0] = L;
      return q;
    }
    const int c = g - 2;
    int f0 = c * C, f1 = (c + 1) * C;
    if (f0 < 1) f0 = 1;
    if (f1 > T - 1) f1 = T - 1;
    q.row0 = f0 * N;
    q.nrows = f1 > f0 ? (f1 - f0) * N : 0;
    int w0 = (c - R) * C, w1 = (c + R + 1) * C;
    if (w0 < 0) w0 = 0;
    if (w1 > T) w1 = T;
    // ranges in increasing order: [anchor 0], window, [anchor T-1]; fixed
    // slots (no dynamic indexing keeps them in registers)
    const bool a0 = w0 > 0, a1 = w1 < T;
    q.seg0[0] = a0 ? 0 : w0 * N;
    q.seg1[0] = a0 ? N : w1 * N;
    q.seg0[1] = a0 ? w0 * N : (T - 1) * N;
    q.seg1[1] = a0 ? w1 * N : L;
    q.seg0[2] = (T - 1) * N;
    q.seg1[2] = L;
    q.nseg = 1 + (a0 ? 1 : 0) + (a1 ? 1 : 0);
    return q;
  }
};

// Locate tile `tile` among the groups (tiles of `rows_per_tile` query rows),
// anchors first (they see every key: longest work first).
__host__ __device__ inline bool find_tile(const Geo& geo, int rows_per_tile, int tile,
                                          QGroup* out, int* row_start) {
  const int ng = geo.n_groups();
  for (int g = 0; g < ng; ++g) {
    QGroup q = geo.group(g);
    const int nt = (q.nrows + rows_per_tile - 1) / rows_per_tile;
    if (tile < nt) {
      *out = q;
      *row_start = q.row0 + tile * rows_per_tile;
      return true;
    }
    tile -= nt;
  }
  return false;
}

__host__ __device__ inline int count_tiles(const Geo& geo, int rows_per_tile) {
  int n = 0;
  for (int g = 0; g < geo.n_groups(); ++g) {
    QGroup q = geo.group(g);
    n += (q.nrows + rows_per_tile - 1) / rows_per_tile;
  }
  return n;
}

}  // namespace vdn
