// aux_kernels.cuh - the memory-bound steps of the SAFE-DiT hot path:
//   * the exact row-constant mask classifier (Eq. (6), per broadcast row),
//   * the context-cache scatter / anchor refresh (Eq. (14), (16), (19)),
//   * the exact tie-stable top-k partition of PCSP (Eq. (12)).
#pragma once

#include "sm100.cuh"

namespace safe {

constexpr int kStatusCheck = 1 << 5;  // SAFE_ERR_DEVICE_CHECK

// ============================================================== classifier

struct ClassifyParams {
  const uint8_t* mask;
  int dtype;  // 0 bool, 1 u8, 2 f32, 3 f16, 4 bf16
  int esize;
  int64_t nb, nh, nq, nk;  // distinct extents (stride-0 dims count once)
  int64_t s0, s1, s2, s3;  // element strides
  unsigned long long* nfail;
  unsigned long long* first_fail;
};

struct RowAcc {
  bool fail;   // a blocked key (bool/u8) or a non-finite entry (float)
  float mn, mx;
};

__device__ __forceinline__ void acc_float(RowAcc& a, float x) {
  if (!isfinite(x)) a.fail = true;
  a.mn = fminf(a.mn, x);
  a.mx = fmaxf(a.mx, x);
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits) { return __uint_as_float(bits << 16); }
__device__ __forceinline__ float f16_bits_to_float(uint32_t bits) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(bits)));
}

__device__ __forceinline__ void acc_elem(RowAcc& a, const uint8_t* p, int dtype) {
  switch (dtype) {
    case 0:
    case 1:
      if (*p == 0) a.fail = true;
      break;
    case 2:
      acc_float(a, *reinterpret_cast<const float*>(p));
      break;
    case 3:
      acc_float(a, f16_bits_to_float(*reinterpret_cast<const uint16_t*>(p)));
      break;
    default:
      acc_float(a, bf16_bits_to_float(*reinterpret_cast<const uint16_t*>(p)));
      break;
  }
}

__device__ __forceinline__ void acc_vec(RowAcc& a, const uint4 v, int dtype) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  if (dtype <= 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if ((w[i] - 0x01010101u) & ~w[i] & 0x80808080u) a.fail = true;  // some byte is zero
  } else if (dtype == 2) {
#pragma unroll
    for (int i = 0; i < 4; ++i) acc_float(a, __uint_as_float(w[i]));
  } else if (dtype == 3) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc_float(a, f16_bits_to_float(w[i] & 0xFFFFu));
      acc_float(a, f16_bits_to_float(w[i] >> 16));
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc_float(a, bf16_bits_to_float(w[i] & 0xFFFFu));
      acc_float(a, bf16_bits_to_float(w[i] >> 16));
    }
  }
}

__global__ void classify_init_kernel(int64_t* result) {
  result[0] = 0;
  result[1] = 0;
  result[2] = INT64_MAX;
}

__global__ void classify_finalize_kernel(int64_t* result) {
  result[0] = result[1] == 0 ? 1 : 0;
  if (result[2] == INT64_MAX) result[2] = -1;
}

// One warp per distinct row; warps stride over rows.
__global__ void __launch_bounds__(256) classify_rows_kernel(const ClassifyParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t rows = p.nb * p.nh * p.nq;
  for (int64_t row = warp_global; row < rows; row += nwarps) {
    const int64_t i = row % p.nq;
    const int64_t bh = row / p.nq;
    const int64_t h = bh % p.nh;
    const int64_t b = bh / p.nh;
    const uint8_t* rp = p.mask + (b * p.s0 + h * p.s1 + i * p.s2) * p.esize;
    RowAcc a{false, INFINITY, -INFINITY};
    if (p.s3 == 1) {
      const int64_t nbytes = p.nk * p.esize;
      const uintptr_t addr = reinterpret_cast<uintptr_t>(rp);
      int64_t head = static_cast<int64_t>((16 - (addr & 15)) & 15);
      if (head > nbytes) head = nbytes;
      const int64_t nvec = (nbytes - head) >> 4;
      const int64_t tail0 = head + (nvec << 4);
      for (int64_t e = lane * p.esize; e < head; e += 32 * p.esize) acc_elem(a, rp + e, p.dtype);
      const uint4* vp = reinterpret_cast<const uint4*>(rp + head);
      int64_t v = lane;
      for (; v + 96 < nvec; v += 128) {
        const uint4 x0 = __ldcs(vp + v), x1 = __ldcs(vp + v + 32), x2 = __ldcs(vp + v + 64),
                    x3 = __ldcs(vp + v + 96);
        acc_vec(a, x0, p.dtype);
        acc_vec(a, x1, p.dtype);
        acc_vec(a, x2, p.dtype);
        acc_vec(a, x3, p.dtype);
      }
      for (; v < nvec; v += 32) acc_vec(a, __ldcs(vp + v), p.dtype);
      for (int64_t e = tail0 + lane * p.esize; e < nbytes; e += 32 * p.esize) acc_elem(a, rp + e, p.dtype);
    } else {
      const int64_t step = p.s3 * p.esize;
      for (int64_t j = lane; j < p.nk; j += 32) acc_elem(a, rp + j * step, p.dtype);
    }
    bool fail = __any_sync(0xffffffffu, a.fail);
    if (p.dtype >= 2) {
      float mn = a.mn, mx = a.mx;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (!(mn == mx)) fail = true;  // finite entries not all equal (-0 == +0)
      if (p.nk == 0) fail = false;
    }
    if (fail && lane == 0) {
      atomicAdd(p.nfail, 1ull);
      atomicMin(p.first_fail, static_cast<unsigned long long>(row));
    }
  }
}

// ============================================================== cache scatter

// Kc[b, S[b,r]] = Ksrc[b, r or S[b,r]] (and V); S == null: full copy.
// One warp per destination row; rows are H*D bf16, moved as 16-byte units.
__global__ void __launch_bounds__(256) cache_scatter_kernel(const uint4* __restrict__ Ksrc,
                                                            const uint4* __restrict__ Vsrc, int src_compact,
                                                            const int32_t* __restrict__ S, int k, uint4* Kc,
                                                            uint4* Vc, int B, int N, int row_units) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t rows = S != nullptr ? static_cast<int64_t>(B) * k : static_cast<int64_t>(B) * N;
  if (row >= rows) return;
  int64_t dst, src;
  if (S != nullptr) {
    const int64_t b = row / k, r = row % k;
    const int idx = __ldg(S + row);
    if (idx < 0 || idx >= N) {
      if (lane == 0) raise_status(kStatusCheck);
      return;
    }
    if (r > 0 && __ldg(S + row - 1) >= idx && lane == 0) raise_status(kStatusCheck);
    dst = b * N + idx;
    src = src_compact ? row : dst;
  } else {
    dst = row;
    src = row;
  }
  const uint4* ks = Ksrc + src * row_units;
  const uint4* vs = Vsrc + src * row_units;
  uint4* kd = Kc + dst * row_units;
  uint4* vd = Vc + dst * row_units;
  int u = lane;
  for (; u + 96 < row_units; u += 128) {
    const uint4 a0 = __ldcs(ks + u), a1 = __ldcs(ks + u + 32), a2 = __ldcs(ks + u + 64), a3 = __ldcs(ks + u + 96);
    const uint4 b0 = __ldcs(vs + u), b1 = __ldcs(vs + u + 32), b2 = __ldcs(vs + u + 64), b3 = __ldcs(vs + u + 96);
    kd[u] = a0; kd[u + 32] = a1; kd[u + 64] = a2; kd[u + 96] = a3;
    vd[u] = b0; vd[u + 32] = b1; vd[u + 64] = b2; vd[u + 96] = b3;
  }
  for (; u < row_units; u += 32) {
    const uint4 a = __ldcs(ks + u), bb = __ldcs(vs + u);
    kd[u] = a;
    vd[u] = bb;
  }
}

// ============================================================== top-k partition

constexpr int kTopkThreads = 1024;

// Order-preserving key: larger float -> larger unsigned key; -0.0 ranks as
// +0.0; NaN is flagged and ranks lowest.
__device__ __forceinline__ uint32_t score_key(float x) {
  if (x != x) {
    raise_status(kStatusCheck);
    return 0u;
  }
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block-wide prefix sum of one int per thread (1024 threads).
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = warp_tot[lane];
    int s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_tot[lane] = s - t;
  }
  __syncthreads();
  const int res = warp_tot[warp] + x - v;
  __syncthreads();
  return res;
}

// Keys of a sample held in shared memory when N is at most this (160 KB of
// keys beside the 32 KB of histograms); larger N read them from global
// memory on every pass.
constexpr int kTopkSmemKeys = 40960;
static_assert(kTopkSmemKeys <= 64 * kTopkThreads, "a thread's segment must fit a 64-bit selection mask");

// One CTA per sample b: radix select of the k-th largest key T (8 bits per
// pass, most significant first), then an ordered compaction: i is selected
// iff key_i > T, or key_i == T and fewer than r earlier indices had key T
// (r = k - #{key > T}); selected indices go to S, the rest to C, both in
// ascending index order. kSmem: the first pass converts the scores once into
// shared memory (loads batched ahead of the histogram updates); the later
// passes and the compaction read the keys from there.
template <bool kSmem>
__global__ void __launch_bounds__(kTopkThreads) topk_partition_kernel(const float* __restrict__ scores, int N, int k,
                                                                      int32_t* __restrict__ S,
                                                                      int32_t* __restrict__ C) {
  constexpr int kBatch = 8;
  extern __shared__ uint32_t topk_keys[];  // [N] when kSmem
  __shared__ int hist[32][256];
  __shared__ int warp_tot[32];
  __shared__ uint32_t sh_prefix;
  __shared__ int sh_remaining;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int b = blockIdx.x;
  const float* sc = scores + static_cast<size_t>(b) * N;
  auto key_at = [&](int i) -> uint32_t {
    if constexpr (kSmem)
      return topk_keys[i];
    else
      return score_key(__ldg(sc + i));
  };

  uint32_t prefix = 0, mask = 0;
  int remaining = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int e = tid; e < 32 * 256; e += kTopkThreads) (&hist[0][0])[e] = 0;
    __syncthreads();
    if (!kSmem || shift == 24) {
      // global scores: kBatch loads in flight before their histogram updates
      for (int base = 0; base < N; base += kBatch * kTopkThreads) {
        float v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int i = base + u * kTopkThreads + tid;
          v[u] = i < N ? __ldg(sc + i) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int i = base + u * kTopkThreads + tid;
          if (i < N) {
            const uint32_t key = score_key(v[u]);
            if constexpr (kSmem) topk_keys[i] = key;
            if ((key & mask) == prefix) atomicAdd(&hist[warp][(key >> shift) & 255u], 1);
          }
        }
      }
    } else {
      for (int i = tid; i < N; i += kTopkThreads) {
        const uint32_t key = topk_keys[i];
        if ((key & mask) == prefix) atomicAdd(&hist[warp][(key >> shift) & 255u], 1);
      }
    }
    __syncthreads();
    // count of digit d = 255 - tid; an exclusive scan over the digits from
    // the top gives, per digit, the number of matching keys above it: the
    // selected digit is the one whose range [above, above + count) holds
    // the remaining-th largest key
    int cnt = 0;
    if (tid < 256) {
#pragma unroll 8
      for (int w = 0; w < 32; ++w) cnt += hist[w][255 - tid];
    }
    const int above = block_exclusive_scan(cnt, warp_tot);
    if (tid < 256 && above < remaining && remaining <= above + cnt) {
      sh_prefix = prefix | (static_cast<uint32_t>(255 - tid) << shift);
      sh_remaining = remaining - above;
    }
    __syncthreads();
    prefix = sh_prefix;
    remaining = sh_remaining;
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t T = prefix;
  const int r = remaining;  // keys equal to T that are selected (lowest indices first)

  // each thread a contiguous segment of indices
  const int seg = (N + kTopkThreads - 1) / kTopkThreads;
  const int i0 = min(N, tid * seg), i1 = min(N, i0 + seg);
  int cnt_gt = 0, cnt_eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at(i);
    cnt_gt += key > T;
    cnt_eq += key == T;
  }
  const int eq_base = block_exclusive_scan(cnt_eq, warp_tot);
  const int take_eq = max(0, min(cnt_eq, r - eq_base));
  const int sel_base = block_exclusive_scan(cnt_gt + take_eq, warp_tot);
  int s_pos = sel_base, c_pos = i0 - sel_base, eq_seen = eq_base;
  int32_t* Sb = S + static_cast<size_t>(b) * k;
  int32_t* Cb = C != nullptr ? C + static_cast<size_t>(b) * (N - k) : nullptr;
  if constexpr (kSmem) {
    // the selection as a bit mask over this thread's segment (at most 40
    // indices), then the key buffer takes the output order: S in [0, k), C
    // in [k, N); both leave by coalesced stores
    uint64_t sel_mask = 0;
    for (int i = i0; i < i1; ++i) {
      const uint32_t key = topk_keys[i];
      bool sel = key > T;
      if (key == T) {
        sel = eq_seen < r;
        ++eq_seen;
      }
      if (sel) sel_mask |= 1ull << (i - i0);
    }
    __syncthreads();  // every key has been read
    c_pos += k;
    for (int i = i0; i < i1; ++i) {
      if ((sel_mask >> (i - i0)) & 1ull)
        topk_keys[s_pos++] = static_cast<uint32_t>(i);
      else
        topk_keys[c_pos++] = static_cast<uint32_t>(i);
    }
    __syncthreads();
    for (int e = tid; e < k; e += kTopkThreads) Sb[e] = static_cast<int32_t>(topk_keys[e]);
    if (Cb != nullptr)
      for (int e = tid; e < N - k; e += kTopkThreads) Cb[e] = static_cast<int32_t>(topk_keys[k + e]);
    return;
  }
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = key_at(i);
    bool sel = key > T;
    if (key == T) {
      sel = eq_seen < r;
      ++eq_seen;
    }
    if (sel) {
      Sb[s_pos++] = i;
    } else if (Cb != nullptr) {
      Cb[c_pos++] = i;
    }
  }
}

// ============================================================== wait self-test

// One CTA waits on an mbarrier that nothing arrives on, with a short limit:
// the bounded wait gives up, raises SAFE_ERR_TIMEOUT in the status word and
// the kernel returns normally.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  mbar_wait(&bar, 0, &abort_flag, limit_ns);
}

}  // namespace safe
