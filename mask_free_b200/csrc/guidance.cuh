// guidance.cuh - the sensitivity field of Eq. (11) and sensitivity-weighted
// classifier-free guidance, Eq. (20), (21).
//
// Sensitivity field s = Norm(G_sigma * s~): the N = grid_h * grid_w PCSP
// scores of a sample lie on the latent token grid in row-major order. The
// Gaussian is separable, so a row pass (into a workspace) is followed by a
// column pass, both with half-sample reflection at the borders; the column
// pass also reduces the per-sample minimum and maximum (as order-preserving
// integer keys, so the atomics are exact and order-free), and a last pass
// maps the field onto [0, 1]. Every output is a short dot product over the
// 2r+1 taps; the three passes move 5 x 4 bytes per token and are latency
// bound at the paper's sizes (N <= 36864 per sample).
//
// SW-CFG: per token, gamma_i = gamma_ctx + (gamma_sens - gamma_ctx) s_i and
// f^ = f_u + gamma_i (f_c - f_u) over the C prediction values of the token;
// one streaming pass (16-byte vectors when the rows allow them).
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace safe {

constexpr int kMaxSmoothRadius = 128;
constexpr int kMaxTaps = 2 * kMaxSmoothRadius + 1;

struct SmoothParams {
  const float* in;     // [B, N] scores
  float* rows;         // [B, N] workspace: row pass
  float* out;          // [B, N] field
  uint32_t* minmax;    // [B, 2] workspace: order-preserving keys of min, max
  int B, gh, gw, r;
  float taps[kMaxTaps];  // G_sigma at -r..r, normalised to sum 1
};

// Index of the half-sample symmetric extension of a line of n values
// (period 2n: ... x1 x0 | x0 ... x_{n-1} | x_{n-1} x_{n-2} ...).
__device__ __forceinline__ int reflect_idx(int i, int n) {
  const int period = 2 * n;
  int m = i % period;
  if (m < 0) m += period;
  return m < n ? m : period - 1 - m;
}

// float <-> uint32 key whose unsigned order is the float order
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Row pass; block 0 of every sample also resets its min / max keys (the
// column pass runs after this kernel on the same stream).
__global__ void smooth_rows_kernel(const __grid_constant__ SmoothParams p) {
  const int b = blockIdx.y;
  const int N = p.gh * p.gw;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    p.minmax[2 * b] = 0xFFFFFFFFu;
    p.minmax[2 * b + 1] = 0u;
  }
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const int y = i / p.gw, x = i - y * p.gw;
  const float* row = p.in + static_cast<size_t>(b) * N + static_cast<size_t>(y) * p.gw;
  float acc = 0.f;
  for (int t = -p.r; t <= p.r; ++t) acc = fmaf(p.taps[t + p.r], __ldg(row + reflect_idx(x + t, p.gw)), acc);
  p.rows[static_cast<size_t>(b) * N + i] = acc;
}

// Column pass and the per-sample min / max.
__global__ void smooth_cols_kernel(const __grid_constant__ SmoothParams p) {
  const int b = blockIdx.y;
  const int N = p.gh * p.gw;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  if (i < N) {
    const int y = i / p.gw, x = i - y * p.gw;
    const float* col = p.rows + static_cast<size_t>(b) * N + x;
    float acc = 0.f;
    for (int t = -p.r; t <= p.r; ++t)
      acc = fmaf(p.taps[t + p.r], col[static_cast<size_t>(reflect_idx(y + t, p.gh)) * p.gw], acc);
    p.out[static_cast<size_t>(b) * N + i] = acc;
    kmin = kmax = order_key(acc);
  }
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xFFFFFFFFu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, o));
  }
  if ((threadIdx.x & 31) == 0) {
    atomicMin(&p.minmax[2 * b], kmin);
    atomicMax(&p.minmax[2 * b + 1], kmax);
  }
}

// Norm: (x - min) / (max - min), 0 for a flat field.
__global__ void norm01_kernel(float* __restrict__ s, const uint32_t* __restrict__ minmax, int N) {
  const int b = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const float lo = key_value(minmax[2 * b]), hi = key_value(minmax[2 * b + 1]);
  float* v = s + static_cast<size_t>(b) * N + i;
  *v = hi > lo ? (*v - lo) / (hi - lo) : 0.f;
}

// Binary variant of Eq. (20): s[b, i] = 1 if i is in S[b] (strictly
// ascending), else 0 - a binary search per token. Out-of-order or
// out-of-range entries of S are flagged.
__global__ void partition_indicator_kernel(const int32_t* __restrict__ S, int k, float* __restrict__ s, int N) {
  const int b = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const int32_t* Sb = S + static_cast<size_t>(b) * k;
  if (i < k) {
    const int v = __ldg(Sb + i);
    if (v < 0 || v >= N || (i + 1 < k && __ldg(Sb + i + 1) <= v)) raise_status(1 << 5);
  }
  int lo = 0, hi = k;  // first position with S >= i
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(Sb + mid) < i) lo = mid + 1;
    else hi = mid;
  }
  s[static_cast<size_t>(b) * N + i] = (lo < k && __ldg(Sb + lo) == i) ? 1.f : 0.f;
}

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ void from_f(float& d, float v) { d = v; }
__device__ __forceinline__ void from_f(__nv_bfloat16& d, float v) { d = __float2bfloat16_rn(v); }

// f^ = f_u + gamma_i (f_c - f_u), gamma_i = gamma_ctx + gamma_diff * s_i.
// VEC values per thread (16 bytes) when C is a multiple of VEC and the
// pointers are 16-byte aligned, else VEC = 1. out may alias f_c or f_u (each
// element is read before it is written, by the same thread).
template <typename T, int VEC>
__global__ void sw_cfg_kernel(const T* fc, const T* fu, const float* __restrict__ s, T* out, size_t n_vec, int C,
                              float gamma_ctx, float gamma_diff) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t v = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < n_vec; v += stride) {
    const size_t e0 = v * VEC;
    const float g = fmaf(gamma_diff, __ldg(s + e0 / C), gamma_ctx);
    if constexpr (VEC == 1) {
      const float c = to_f(fc[e0]), u = to_f(fu[e0]);
      from_f(out[e0], fmaf(g, c - u, u));
    } else {
      union Pack {
        uint4 v;
        T e[VEC];
      } cv, uv, ov;
      cv.v = *reinterpret_cast<const uint4*>(fc + e0);
      uv.v = *reinterpret_cast<const uint4*>(fu + e0);
#pragma unroll
      for (int q = 0; q < VEC; ++q) {
        const float c = to_f(cv.e[q]), u = to_f(uv.e[q]);
        from_f(ov.e[q], fmaf(g, c - u, u));
      }
      *reinterpret_cast<uint4*>(out + e0) = ov.v;
    }
  }
}

}  // namespace safe
