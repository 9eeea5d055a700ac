// cross_attn.cuh - image->text cross-attention with the text padding kept as
// per-sample valid key lengths (Eq. (4), Eq. (17)), and the per-head PCSP
// partial scores built from the same probabilities (Eq. (9), (10)).
//
// All M <= 256 text keys of a (b, h) fit one tile, so the softmax is exact in
// one pass. One CTA (4 warps) owns one 128-row query tile of one (b, h):
//   1. TMA loads the query tile (dense rows, or rows of S via gather4);
//   2. the CTA copies the first Lp = ceil32(valid_len) text key / value rows
//      into the swizzled shared-memory layout the tensor core reads, writing
//      zeros for rows >= valid_len (padding rows are never read, so they may
//      hold any bytes);
//   3. S = Q Ky^T (M=128, N=Lp) into TMEM; each thread owns one query row:
//      max over valid keys, p = 2^(s*scale*log2(e) - max), l = sum p,
//      score = sum_j w_j p_j / l (the PCSP partial for this head);
//   4. P (bf16) goes back into TMEM and O = P Vy / l is written as bf16.
#pragma once

#include "flash_attn.cuh"

namespace safe {

struct CrossParams {
  CUtensorMap q_map[2];   // 4-D dense Q map per chunk
  CUtensorMap qg_map[2];  // 2-D gather map per chunk
  const __nv_bfloat16* Ky;  // [B, M, H, D]
  const __nv_bfloat16* Vy;
  const int32_t* valid_len;  // [B]
  const int32_t* q_idx;      // [B, nq] or null
  const float* w;            // [B, M] or null (uniform on valid keys)
  __nv_bfloat16* O;          // [B, nq, H, D] or null
  float* partial;            // [B, H, nq] or null
  int B, N, M, H, nq;
  float scale_log2;
  int gather;
};

constexpr int kCrossThreads = 128;

template <int D>
__host__ __device__ constexpr int cross_smem_bytes(int M) {
  return 1024 + TileCfg<D>::kTileBytes + 2 * (((M + 31) / 32) * 32) * D * 2 + 256 * 4 + 64;
}

__host__ __device__ constexpr int cross_tmem_cols(int M, int D) {
  return ((M <= 128 ? 128 : 256) + D) <= 256 ? 256 : 512;
}

template <int D>
__global__ void __launch_bounds__(kCrossThreads) cross_attn_kernel(const __grid_constant__ CrossParams p) {
  using C = TileCfg<D>;
  constexpr int TB = C::kTileBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int Mp = ((p.M + 31) / 32) * 32;
  uint8_t* sQ = sm;
  uint8_t* sKy = sQ + TB;
  uint8_t* sVy = sKy + Mp * D * 2;
  float* sw = reinterpret_cast<float*>(sVy + Mp * D * 2);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sw + 256);
  uint64_t* q_full = bars;
  uint64_t* s_bar = bars + 1;
  uint64_t* o_bar = bars + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.z, h = blockIdx.y;
  const int q0 = blockIdx.x * 128;
  const int s_region = p.M <= 128 ? 128 : 256;
  const uint32_t tcols = static_cast<uint32_t>(cross_tmem_cols(p.M, D));

  int L = __ldg(p.valid_len + b);
  if (L < 1 || L > p.M) {
    if (tid == 0) raise_status(1 << 5);
    L = L < 1 ? 1 : p.M;
  }
  const int Lp = ((L + 31) / 32) * 32;

  if (tid == 0) {
    abort_flag = 0;
    mbar_init(q_full, 1);
    mbar_init(s_bar, 1);
    mbar_init(o_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, tcols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  // 1. query tile
  if (warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(q_full, TB);
    __syncwarp();
    if (!p.gather) {
      if (lane == 0)
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(sQ + C::chunk_off(c), &p.q_map[c], q_full, 64 * c, h, q0, b);
    } else {
      int y[4];
      for (int u = 0; u < 4; ++u) {
        int r = q0 + 4 * lane + u;
        r = r < p.nq ? r : p.nq - 1;
        int idx = __ldg(p.q_idx + static_cast<size_t>(b) * p.nq + r);
        if (idx < 0 || idx >= p.N) {
          raise_status(1 << 5);
          idx = 0;
        }
        y[u] = b * p.N + idx;
      }
      for (int c = 0; c < C::kChunks; ++c)
        tma_gather4(sQ + C::chunk_off(c) + 4 * lane * C::row_bytes(c), &p.qg_map[c], q_full, h * D + 64 * c, y[0],
                    y[1], y[2], y[3]);
    }
  }

  // 2. text keys / values -> swizzled shared memory (zeros past valid_len)
  {
    constexpr int kUnits = D / 8;  // 16-byte units per row
    const size_t row_stride = static_cast<size_t>(p.H) * D;  // elements between text tokens
    const __nv_bfloat16* kbase = p.Ky + (static_cast<size_t>(b) * p.M * p.H + h) * D;
    const __nv_bfloat16* vbase = p.Vy + (static_cast<size_t>(b) * p.M * p.H + h) * D;
    for (int e = tid; e < Lp * kUnits; e += kCrossThreads) {
      const int r = e / kUnits, u = e % kUnits;
      const int c = u >> 3, uc = u & 7;  // chunk and unit within the chunk row
      uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      if (r < L) {
        kv = __ldg(reinterpret_cast<const uint4*>(kbase + r * row_stride) + u);
        if (p.O != nullptr) vv = __ldg(reinterpret_cast<const uint4*>(vbase + r * row_stride) + u);
      }
      const int rb = C::row_bytes(c);
      const int xr = (rb == 128) ? (r & 7) : ((r >> 1) & 3);  // 128B / 64B swizzle phase of row r
      const uint32_t off = static_cast<uint32_t>(c) * Mp * 128 + r * rb + ((uc ^ xr) << 4);
      *reinterpret_cast<uint4*>(sKy + off) = kv;
      *reinterpret_cast<uint4*>(sVy + off) = vv;
    }
    for (int j = tid; j < Lp; j += kCrossThreads) {
      float wj = 0.f;
      if (j < L) wj = p.w != nullptr ? __ldg(p.w + static_cast<size_t>(b) * p.M + j) : 1.f / static_cast<float>(L);
      sw[j] = wj;
    }
  }
  fence_proxy_async_smem();
  __syncthreads();

  // 3. S = Q Ky^T
  if (tid == 0) {
    if (mbar_wait(q_full, 0, &abort_flag)) {
      tc_fence_after();
      const uint32_t idS = make_idesc_bf16(128, Lp, 0, 0);
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sKy);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int c = kk >> 2;
        const uint64_t bd = make_sdesc(aK + c * Mp * 128 + (kk & 3) * 32, 16, 8 * C::row_bytes(c), C::swizzle(c));
        umma_ss(tbase, kmajor_desc<D>(aQ, kk), bd, idS, kk > 0 ? 1u : 0u);
      }
      umma_commit(s_bar);
    } else {
      mbar_wait_drain(q_full, 0);
    }
  }

  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tbase + lane_addr;
  const uint32_t tO = tbase + lane_addr + s_region;
  const int q_row = q0 + row;
  const bool valid = q_row < p.nq;
  const float sl2 = p.scale_log2;
  bool ok = __all_sync(0xffffffffu, mbar_wait(s_bar, 0, &abort_flag));
  float l = 0.f, score = 0.f;
  if (ok) {
    tc_fence_after();
    // pass 1: row max over valid keys
    float mx = -INFINITY;
    for (int c = 0; c < Lp / 32; ++c) {
      uint32_t sr[32];
      tmem_ld32(tS + 32 * c, sr);
      tmem_ld_wait32(sr);
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (32 * c + i < L) mx = fmaxf(mx, __uint_as_float(sr[i]));
    }
    const float neg = -mx * sl2;
    // pass 2: probabilities, sums, P -> TMEM
    for (int c = 0; c < Lp / 32; ++c) {
      uint32_t sr[32];
      tmem_ld32(tS + 32 * c, sr);
      tmem_ld_wait32(sr);
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int j0 = 32 * c + 2 * i;
        const float a = j0 < L ? ex2_approx(fmaf(__uint_as_float(sr[2 * i]), sl2, neg)) : 0.f;
        const float bb = j0 + 1 < L ? ex2_approx(fmaf(__uint_as_float(sr[2 * i + 1]), sl2, neg)) : 0.f;
        l += a + bb;
        score = fmaf(sw[j0], a, score);
        score = fmaf(sw[j0 + 1], bb, score);
        pk[i] = pack_bf16x2(a, bb);
      }
      if (p.O != nullptr) tmem_st16(tS + 16 * c, pk);
    }
    if (p.partial != nullptr && valid)
      p.partial[(static_cast<size_t>(b) * p.H + h) * p.nq + q_row] = score / l;
  }

  // 4. O = P Vy / l
  if (p.O != nullptr) {
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && ok && !abort_flag) {
      tc_fence_after();
      constexpr uint32_t idPV0 = make_idesc_bf16(128, C::width(0), 0, 1);
      constexpr uint32_t idPV1 = make_idesc_bf16(128, C::kChunks > 1 ? C::width(1) : 64, 0, 1);
      const uint32_t aV = smem_u32(sVy);
      for (int kk = 0; kk < Lp / 16; ++kk) {
        const uint32_t acc = kk > 0 ? 1u : 0u;
        umma_ts(tbase + s_region, tbase + kk * 8,
                make_sdesc(aV + kk * 16 * C::row_bytes(0), 16, 8 * C::row_bytes(0), C::swizzle(0)), idPV0, acc);
        if (C::kChunks > 1)
          umma_ts(tbase + s_region + 64, tbase + kk * 8,
                  make_sdesc(aV + Mp * 128 + kk * 16 * C::row_bytes(1), 16, 8 * C::row_bytes(1), C::swizzle(1)),
                  idPV1, acc);
      }
      umma_commit(o_bar);
    }
    ok = ok && __all_sync(0xffffffffu, mbar_wait(o_bar, 0, &abort_flag));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      __nv_bfloat16* orow = p.O + ((static_cast<size_t>(b) * p.nq + (valid ? q_row : 0)) * p.H + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_ld_wait32(o);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, tcols);
}

// scores[b, i] (+)= (1/H) * sum_h partial[b, h, i], heads summed in order.
__global__ void pcsp_reduce_kernel(const float* __restrict__ partial, float* __restrict__ scores, int B, int H, int N,
                                   int accumulate) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int b = blockIdx.y;
  if (i >= N) return;
  float acc = 0.f;
  for (int h = 0; h < H; ++h) acc += partial[(static_cast<size_t>(b) * H + h) * N + i];
  acc = acc / static_cast<float>(H);
  float* dst = scores + static_cast<size_t>(b) * N + i;
  *dst = accumulate ? *dst + acc : acc;
}

}  // namespace safe
