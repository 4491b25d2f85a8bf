// layout.cuh -- where row n of head h of batch entry b starts in a tensor whose
// last (head-dimension) axis is contiguous: element offset b*sb + h*sh + n*sn.
// [B, H, N, d] contiguous is (H*N*d, N*d, d); [B, N, H, d] ("BSHD") seen as
// [B, H, N, d] is (N*H*d, d, H*d).
#pragma once

namespace fa {

struct Strides {
  long long b, h, n;  // elements between consecutive batch entries, heads, rows
  __host__ __device__ __forceinline__ long long row(int bi, int hi, int ni) const {
    return bi * b + hi * h + static_cast<long long>(ni) * n;
  }
};

__host__ __device__ __forceinline__ Strides contiguous_strides(int heads, int N, int d) {
  return Strides{static_cast<long long>(heads) * N * d, static_cast<long long>(N) * d, d};
}

}  // namespace fa
