// simt_f32.cuh -- fp32 attention forward and backward on CUDA cores.
//
// The fp32 path keeps every product, exponential and sum in fp32 (tensor-core
// TF32 would not meet a 1e-5 bound).  One warp owns one output row; its lanes
// split the head dimension and reduce dot products with butterfly shuffles (all
// lanes end with the identical sum, so the softmax state stays warp-uniform).
// Key/value (or query/dO) rows are staged through shared memory, 32 at a time.
//
// Forward: online softmax over the allowed keys, one key at a time ("Flash
// attention and efficient attention", "Derivation: Incremental Softmax": safe
// softmax, and the Step 3 rescale whenever a new row maximum arrives).
// Backward: S and P are recomputed from Q, K and the saved logsumexp ("Backward
// Pass: Recomputation"); dQ is owned by query-row warps and dK/dV by key-row
// warps, so nothing is accumulated with atomics and every result is
// deterministic.
#pragma once

#include <stdint.h>

#include "layout.cuh"

namespace fa {

struct SimtParams {
  const float* q;
  const float* k;
  const float* v;
  const float* o;
  const float* dout;
  const float* lse;
  float* o_out;
  float* lse_out;
  float* dq;
  float* dk;
  float* dv;
  float* Drow;  // workspace: D_i = sum_k dO_ik O_ik, [B*H*N]
  int B, H, Hkv, N, g;
  float scale;
  int causal, window;
  const uint8_t* bmask;  // optional 0/1 mask per 128 x 128 block, [head][nbt][nbt]
  long long bmask_hs;    // elements between heads' masks (0: shared)
  int nbt;               // ceil(N / 128)
  const int* seqlens;    // optional valid rows per batch entry (padded layout)
  // element strides (batch, head, row) of each [B, heads, N, D] tensor; o is
  // also the layout of o_out
  Strides sq, sk, sv, so, sdo, sdq, sdk, sdv;
};

__device__ __forceinline__ int simt_valid_rows(const SimtParams& p, int b) {
  return p.seqlens ? max(0, min(p.seqlens[b], p.N)) : p.N;
}

__device__ __forceinline__ bool keep_ij(int i, int j, int causal, int window) {
  return (!causal || j <= i) && (window < 0 || abs(i - j) <= window);
}

// keep_ij and, under a block mask, block (i / 128, j / 128) of query head bh on.
__device__ __forceinline__ bool keep_ijb(const SimtParams& p, int bh, int i, int j) {
  if (!keep_ij(i, j, p.causal, p.window)) return false;
  return !p.bmask || p.bmask[bh * p.bmask_hs + static_cast<long long>(i >> 7) * p.nbt + (j >> 7)] != 0;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

constexpr int kSimtRows = 8;  // warps (rows) per block
constexpr int kSimtTile = 32;  // staged rows per smem tile

// Keys that query rows [r0, r1) may see: [lo, hi).
__device__ __forceinline__ void simt_key_range(int r0, int r1, int N, int causal, int window, int& lo, int& hi) {
  lo = 0;
  hi = N;
  if (causal) hi = min(hi, r1);
  if (window >= 0) {
    lo = max(lo, r0 - window);
    hi = min(hi, r1 + window);
  }
}
// Query rows that keys [c0, c1) are seen by: [lo, hi).
__device__ __forceinline__ void simt_query_range(int c0, int c1, int N, int causal, int window, int& lo, int& hi) {
  lo = 0;
  hi = N;
  if (causal) lo = max(lo, c0);
  if (window >= 0) {
    lo = max(lo, c0 - window);
    hi = min(hi, c1 + window);
  }
}

template <int D>
__global__ void __launch_bounds__(256) fwd_simt_f32_kernel(const SimtParams p) {
  constexpr int E = D / 32;
  __shared__ float sK[kSimtTile][D];
  __shared__ float sV[kSimtTile][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
  const int kh = h / p.g;
  const int Lb = simt_valid_rows(p, b);
  const int r0 = blockIdx.x * kSimtRows, r1 = min(Lb, r0 + kSimtRows);
  const int i = r0 + warp;
  const bool active = i < Lb;
  const float* qrow = p.q + p.sq.row(b, h, active ? i : 0);
  const float* kbase = p.k + p.sk.row(b, kh, 0);
  const float* vbase = p.v + p.sv.row(b, kh, 0);
  float q[E], acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    q[e] = qrow[lane + 32 * e];
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  int lo, hi;
  simt_key_range(r0, max(r0, r1), Lb, p.causal, p.window, lo, hi);
  for (int kt = lo; kt < hi; kt += kSimtTile) {
    const int cnt = min(kSimtTile, hi - kt);
    __syncthreads();
    for (int x = threadIdx.x; x < cnt * D; x += blockDim.x) {
      sK[x / D][x % D] = kbase[static_cast<long long>(kt + x / D) * p.sk.n + x % D];
      sV[x / D][x % D] = vbase[static_cast<long long>(kt + x / D) * p.sv.n + x % D];
    }
    __syncthreads();
    if (!active) continue;
    for (int jj = 0; jj < cnt; ++jj) {
      const int j = kt + jj;
      if (!keep_ijb(p, bh, i, j)) continue;
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) s = fmaf(q[e], sK[jj][lane + 32 * e], s);
      s = warp_sum(s) * p.scale;
      if (s > m) {  // a new row maximum: rescale what was accumulated
        const float a = expf(m - s);
        l *= a;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] *= a;
        m = s;
      }
      const float pe = expf(s - m);
      l += pe;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = fmaf(pe, sV[jj][lane + 32 * e], acc[e]);
    }
  }
  if (i >= p.N) return;  // padded rows (i >= Lb) end with l = 0: O = 0, LSE = -inf
  const float inv = l > 0.f ? 1.f / l : 0.f;
  float* orow = p.o_out + p.so.row(b, h, i);
#pragma unroll
  for (int e = 0; e < E; ++e) orow[lane + 32 * e] = acc[e] * inv;
  if (lane == 0) p.lse_out[static_cast<size_t>(bh) * p.N + i] = l > 0.f ? m + logf(l) : -INFINITY;
}

// D_i = sum_k dO_ik O_ik (equal to sum_j P_ij dP_ij, the softmax-Jacobian row term).
template <int D>
__global__ void __launch_bounds__(256) bwd_rowdot_f32_kernel(const SimtParams p) {
  constexpr int E = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row = static_cast<size_t>(blockIdx.x) * kSimtRows + warp;
  if (row >= static_cast<size_t>(p.B) * p.H * p.N) return;
  const int n = static_cast<int>(row % p.N);
  const int b = static_cast<int>(row / (static_cast<size_t>(p.H) * p.N));
  const int h = static_cast<int>((row / p.N) % p.H);
  const float* dorow = p.dout + p.sdo.row(b, h, n);
  const float* orow = p.o + p.so.row(b, h, n);
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) s = fmaf(dorow[lane + 32 * e], orow[lane + 32 * e], s);
  s = warp_sum(s);
  if (lane == 0) p.Drow[row] = n < simt_valid_rows(p, b) ? s : 0.f;
}

// dK, dV: one warp per key row of a kv head, summing over its query heads.
template <int D>
__global__ void __launch_bounds__(256) bwd_dkdv_f32_kernel(const SimtParams p) {
  constexpr int E = D / 32;
  __shared__ float sQ[kSimtTile][D];
  __shared__ float sO[kSimtTile][D];  // dO rows
  __shared__ float sL[kSimtTile], sD[kSimtTile];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bkv = blockIdx.y, b = bkv / p.Hkv, kh = bkv % p.Hkv;
  const int Lb = simt_valid_rows(p, b);
  const int c0 = blockIdx.x * kSimtRows, c1 = min(Lb, c0 + kSimtRows);
  const int j = c0 + warp;
  const bool active = j < Lb;
  const float* krow = p.k + p.sk.row(b, kh, active ? j : 0);
  const float* vrow = p.v + p.sv.row(b, kh, active ? j : 0);
  float kk[E], vv[E], dk[E], dv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    kk[e] = krow[lane + 32 * e];
    vv[e] = vrow[lane + 32 * e];
    dk[e] = 0.f;
    dv[e] = 0.f;
  }
  int lo, hi;
  simt_query_range(c0, max(c0, c1), Lb, p.causal, p.window, lo, hi);
  for (int hq = 0; hq < p.g; ++hq) {
    const int bh = b * p.H + kh * p.g + hq;
    const float* qbase = p.q + p.sq.row(b, kh * p.g + hq, 0);
    const float* obase = p.dout + p.sdo.row(b, kh * p.g + hq, 0);
    for (int it = lo; it < hi; it += kSimtTile) {
      const int cnt = min(kSimtTile, hi - it);
      __syncthreads();
      for (int x = threadIdx.x; x < cnt * D; x += blockDim.x) {
        sQ[x / D][x % D] = qbase[static_cast<long long>(it + x / D) * p.sq.n + x % D];
        sO[x / D][x % D] = obase[static_cast<long long>(it + x / D) * p.sdo.n + x % D];
      }
      for (int x = threadIdx.x; x < cnt; x += blockDim.x) {
        sL[x] = p.lse[static_cast<size_t>(bh) * p.N + it + x];
        sD[x] = p.Drow[static_cast<size_t>(bh) * p.N + it + x];
      }
      __syncthreads();
      if (!active) continue;
      for (int ii = 0; ii < cnt; ++ii) {
        const int i = it + ii;
        if (!keep_ijb(p, bh, i, j)) continue;
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          s = fmaf(sQ[ii][lane + 32 * e], kk[e], s);
          dp = fmaf(sO[ii][lane + 32 * e], vv[e], dp);
        }
        s = warp_sum(s) * p.scale;
        dp = warp_sum(dp);
        const float pr = expf(s - sL[ii]);
        const float ds = pr * (dp - sD[ii]);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          dv[e] = fmaf(pr, sO[ii][lane + 32 * e], dv[e]);
          dk[e] = fmaf(ds, sQ[ii][lane + 32 * e], dk[e]);
        }
      }
    }
  }
  if (j >= p.N) return;  // padded keys (j >= Lb) keep dk = dv = 0
  float* dkrow = p.dk + p.sdk.row(b, kh, j);
  float* dvrow = p.dv + p.sdv.row(b, kh, j);
#pragma unroll
  for (int e = 0; e < E; ++e) {
    dkrow[lane + 32 * e] = dk[e] * p.scale;
    dvrow[lane + 32 * e] = dv[e];
  }
}

// dQ: one warp per query row.
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_f32_kernel(const SimtParams p) {
  constexpr int E = D / 32;
  __shared__ float sK[kSimtTile][D];
  __shared__ float sV[kSimtTile][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, b = bh / p.H, h = bh % p.H;
  const int kh = h / p.g;
  const int Lb = simt_valid_rows(p, b);
  const int r0 = blockIdx.x * kSimtRows, r1 = min(Lb, r0 + kSimtRows);
  const int i = r0 + warp;
  const bool active = i < Lb;
  const int ir = i < p.N ? i : 0;
  const size_t row = static_cast<size_t>(bh) * p.N + ir;  // LSE and D rows (contiguous)
  float q[E], dO[E], dq[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    q[e] = p.q[p.sq.row(b, h, ir) + lane + 32 * e];
    dO[e] = p.dout[p.sdo.row(b, h, ir) + lane + 32 * e];
    dq[e] = 0.f;
  }
  const float L = p.lse[row], Dr = p.Drow[row];
  const float* kbase = p.k + p.sk.row(b, kh, 0);
  const float* vbase = p.v + p.sv.row(b, kh, 0);
  int lo, hi;
  simt_key_range(r0, max(r0, r1), Lb, p.causal, p.window, lo, hi);
  for (int kt = lo; kt < hi; kt += kSimtTile) {
    const int cnt = min(kSimtTile, hi - kt);
    __syncthreads();
    for (int x = threadIdx.x; x < cnt * D; x += blockDim.x) {
      sK[x / D][x % D] = kbase[static_cast<long long>(kt + x / D) * p.sk.n + x % D];
      sV[x / D][x % D] = vbase[static_cast<long long>(kt + x / D) * p.sv.n + x % D];
    }
    __syncthreads();
    if (!active) continue;
    for (int jj = 0; jj < cnt; ++jj) {
      const int j = kt + jj;
      if (!keep_ijb(p, bh, i, j)) continue;
      float s = 0.f, dp = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        s = fmaf(q[e], sK[jj][lane + 32 * e], s);
        dp = fmaf(dO[e], sV[jj][lane + 32 * e], dp);
      }
      s = warp_sum(s) * p.scale;
      dp = warp_sum(dp);
      const float ds = expf(s - L) * (dp - Dr);
#pragma unroll
      for (int e = 0; e < E; ++e) dq[e] = fmaf(ds, sK[jj][lane + 32 * e], dq[e]);
    }
  }
  if (i >= p.N) return;  // padded rows (i >= Lb) keep dq = 0
#pragma unroll
  for (int e = 0; e < E; ++e) p.dq[p.sdq.row(b, h, i) + lane + 32 * e] = dq[e] * p.scale;
}

}  // namespace fa
