// Streaming kept rows by column slices, and the deterministic sum of a few partial rows.
//
// The sparse product y = sum over kept rows r of x_r * Wt[r][:] ("Spark Transformer",
// section 3.1, SVMM, read with the input-major weight so that a kept row is one run) is
// split over a CTA grid in two dimensions: CG column groups x RG row groups. CTA (cg, rg)
// reads, for every kept row of rank r = rg (mod RG), the slice of its columns that column
// group cg owns, and sums them into a partial row of those columns. Each column then has RG
// partial sums only (not one per CTA), and the last of a column group's RG CTAs to finish
// adds them in row-group order: no grid barrier and no all-to-all reduction, and the result
// does not depend on timing. Within a CTA, thread t takes vector v0 + t % nv of the rows
// t / nv, t / nv + R, ... (R = 1024 / nv rows per pass), U rows in flight, and the passes'
// sums are added in a fixed order through shared memory.
#pragma once

#include "common.cuh"

namespace wina {

constexpr int kCT = 1024;  // threads per CTA of the column-slice stream

// Column slice [v0, v0 + nv) (16-byte vectors, nv <= kCT) of rows row_of(i), i < cnt,
// times val_of(i), summed. On return thread t < nv holds the sum of vector v0 + t in out
// (EPV floats); red: shared memory of at least kCT * 4 floats. Every thread must call it.
template <bool BF16, int U, typename RowOf, typename ValOf>
__device__ __forceinline__ void stream_cols(const void* __restrict__ Wt, int64_t V, int v0, int nv, int cnt,
                                            RowOf row_of, ValOf val_of, float* red, uint64_t pol,
                                            float (&out)[VecOps<BF16>::EPV]) {
  constexpr int EPV = VecOps<BF16>::EPV;
  const int t = threadIdx.x;
  const int R = kCT / nv;
  const int ph = t / nv;
  const uint4* col = reinterpret_cast<const uint4*>(Wt) + v0 + (t % nv);
  float acc[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) acc[e] = 0.f;
  if (ph < R) {
    int i = ph;
    for (; i + (U - 1) * R < cnt; i += U * R) {
      uint4 w[U];
      float x[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        x[u] = val_of(i + u * R);
        w[u] = ld_stream_u4(col + (int64_t)row_of(i + u * R) * V, pol);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) VecOps<BF16>::fma(acc, w[u], x[u]);
    }
    for (; i < cnt; i += R) VecOps<BF16>::fma(acc, ld_stream_u4(col + (int64_t)row_of(i) * V, pol), val_of(i));
  }
  // the R passes' sums of each vector, in pass order, 4 floats at a time
#pragma unroll
  for (int h = 0; h < EPV; h += 4) {
    __syncthreads();
    reinterpret_cast<float4*>(red)[t] = make_float4(acc[h], acc[h + 1], acc[h + 2], acc[h + 3]);
    __syncthreads();
    if (t < nv) {
      float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int p = 0; p < R; ++p) {
        const float4 v = reinterpret_cast<const float4*>(red)[p * nv + t];
        s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
      }
      out[h] = s.x, out[h + 1] = s.y, out[h + 2] = s.z, out[h + 3] = s.w;
    }
  }
  __syncthreads();
}

// Arrival of this CTA at its column group's counter (after its partial row's stores):
// true for the last of the group's RG CTAs, which then resets the counter for the next
// call and may read the others' partial rows. Every thread must call it.
__device__ __forceinline__ bool group_arrive_last(unsigned* counter, int RG) {
  __shared__ int s_last;
  __syncthreads();  // this CTA's partial stores are done
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned old = atomicAdd(counter, 1u);
    const int last = old == (unsigned)(RG - 1);
    if (last) {
      atomicExch(counter, 0u);
      __threadfence();  // the other CTAs' partial rows are visible to this CTA's reads below
    }
    s_last = last;
  }
  __syncthreads();
  return s_last != 0;
}

}  // namespace wina
