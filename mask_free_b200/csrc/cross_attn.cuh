// cross_attn.cuh - image->text cross-attention with the text padding kept as
// per-sample valid key lengths (Eq. (4), Eq. (17)), and the per-head PCSP
// partial scores built from the same probabilities (Eq. (9), (10)).
//
// All M <= 256 text keys of a (b, h) fit one tile, so the softmax is exact in
// one pass over them. A few CTAs (4 warps each) share the query tiles of one
// (b, h); each CTA
//   1. copies the first Lp = ceil32(valid_len) text key / value rows into the
//      swizzled shared-memory layout the tensor core reads, once, writing
//      zeros for rows >= valid_len (padding rows are never read, so they may
//      hold any bytes), with all of a thread's loads in flight together;
//   2. streams its range of 128-row query tiles through a two-buffer TMA
//      ring (dense rows, or rows of S via gather4), the next tile's load in
//      flight while the current one is processed;
//   3. per tile: S = Q Ky^T (M=128, N=Lp) into TMEM; each thread owns one
//      query row: max over valid keys, p = 2^(s*scale*log2(e) - max),
//      l = sum p, score = sum_j w_j p_j / l (the PCSP partial for this head);
//      P (bf16) goes back into TMEM and O = P Vy / l is written as bf16.
// Two CTAs fit an SM (M <= 128), so one CTA's softmax overlaps the other's
// loads and MMAs.
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
  return 1024 + 2 * TileCfg<D>::kTileBytes + 2 * (((M + 31) / 32) * 32) * D * 2 + 256 * 4 + 64;
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
  uint8_t* sQ = sm;  // two query-tile buffers
  uint8_t* sKy = sQ + 2 * TB;
  uint8_t* sVy = sKy + Mp * D * 2;
  float* sw = reinterpret_cast<float*>(sVy + Mp * D * 2);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sw + 256);
  uint64_t* q_full = bars;      // [2]
  uint64_t* s_bar = bars + 2;
  uint64_t* o_bar = bars + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.z, h = blockIdx.y;
  const int n_tiles = (p.nq + 127) / 128;
  const int per = (n_tiles + gridDim.x - 1) / gridDim.x;
  const int tile0 = blockIdx.x * per;
  const int tile1 = tile0 + per < n_tiles ? tile0 + per : n_tiles;
  if (tile0 >= tile1) return;  // uniform for the CTA, before any barrier or TMEM use
  const int n_my = tile1 - tile0;
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
    mbar_init(&q_full[0], 1);
    mbar_init(&q_full[1], 1);
    mbar_init(s_bar, 1);
    mbar_init(o_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, tcols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  // query tile `it` of this CTA -> buffer it & 1 (issued by warp 0)
  int q_issued = 0;
  auto load_q = [&](int it) {
    const int buf = it & 1;
    q_issued = it + 1;
    const int q0 = (tile0 + it) * 128;
    if (lane == 0) mbar_arrive_expect_tx(&q_full[buf], TB);
    __syncwarp();
    if (!p.gather) {
      if (lane == 0)
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(sQ + buf * TB + C::chunk_off(c), &p.q_map[c], &q_full[buf], 64 * c, h, q0, b);
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
        tma_gather4(sQ + buf * TB + C::chunk_off(c) + 4 * lane * C::row_bytes(c), &p.qg_map[c], &q_full[buf],
                    h * D + 64 * c, y[0], y[1], y[2], y[3]);
    }
  };
  if (warp == 0) {
    load_q(0);
    if (n_my > 1) load_q(1);
  }

  // text keys / values -> swizzled shared memory (zeros past valid_len);
  // eight 16-byte units per thread are loaded before any is stored
  {
    constexpr int kUnits = D / 8;  // 16-byte units per row
    const size_t row_stride = static_cast<size_t>(p.H) * D;  // elements between text tokens
    const __nv_bfloat16* kbase = p.Ky + (static_cast<size_t>(b) * p.M * p.H + h) * D;
    const __nv_bfloat16* vbase = p.Vy + (static_cast<size_t>(b) * p.M * p.H + h) * D;
    const int total = Lp * kUnits;
    for (int e0 = tid; e0 < total; e0 += 8 * kCrossThreads) {
      uint4 kv[8], vv[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int e = e0 + k * kCrossThreads;
        const int r = e / kUnits, u = e % kUnits;
        kv[k] = make_uint4(0, 0, 0, 0);
        vv[k] = make_uint4(0, 0, 0, 0);
        if (e < total && r < L) {
          kv[k] = __ldg(reinterpret_cast<const uint4*>(kbase + r * row_stride) + u);
          if (p.O != nullptr) vv[k] = __ldg(reinterpret_cast<const uint4*>(vbase + r * row_stride) + u);
        }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int e = e0 + k * kCrossThreads;
        if (e >= total) break;
        const int r = e / kUnits, u = e % kUnits;
        // K (K-major operand): 64-wide chunks, 128B swizzle (+ a 32-wide,
        // 64B-swizzled tail chunk for D = 96)
        const int c = u >> 3, uc = u & 7;
        const int rb = C::row_bytes(c);
        const int xr = (rb == 128) ? (r & 7) : ((r >> 1) & 3);  // swizzle phase of row r
        *reinterpret_cast<uint4*>(sKy + static_cast<uint32_t>(c) * Mp * 128 + r * rb + ((uc ^ xr) << 4)) = kv[k];
        // V (MN-major operand of P V): 32-wide chunks, 64B swizzle, so one
        // N = D instruction covers the head dim
        const int vc = u >> 2, vu = u & 3;
        *reinterpret_cast<uint4*>(sVy + static_cast<uint32_t>(vc) * Mp * 64 + r * 64 + ((vu ^ ((r >> 1) & 3)) << 4)) =
            vv[k];
      }
    }
    for (int j = tid; j < Lp; j += kCrossThreads) {
      float wj = 0.f;
      if (j < L) wj = p.w != nullptr ? __ldg(p.w + static_cast<size_t>(b) * p.M + j) : 1.f / static_cast<float>(L);
      sw[j] = wj;
    }
  }
  fence_proxy_async_smem();
  __syncthreads();

  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t tS = tbase + lane_addr;
  const uint32_t tO = tbase + lane_addr + s_region;
  const float sl2 = p.scale_log2;
  const uint32_t idS = make_idesc_bf16(128, Lp, 0, 0);
  constexpr uint32_t idPV = make_idesc_bf16(128, D, 0, 1);
  const uint32_t aK = smem_u32(sKy), aV = smem_u32(sVy);

  bool ok = true;
  for (int it = 0; it < n_my && ok; ++it) {
    const int buf = it & 1;
    const int q_row = (tile0 + it) * 128 + row;
    const bool valid = q_row < p.nq;
    // S = Q Ky^T
    if (tid == 0) {
      if (mbar_wait(&q_full[buf], (it >> 1) & 1, &abort_flag)) {
        tc_fence_after();
        const uint32_t aQ = smem_u32(sQ + buf * TB);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk >> 2;
          const uint64_t bd = make_sdesc(aK + c * Mp * 128 + (kk & 3) * 32, 16, 8 * C::row_bytes(c), C::swizzle(c));
          umma_ss(tbase, kmajor_desc<D>(aQ, kk), bd, idS, kk > 0 ? 1u : 0u);
        }
        umma_commit(s_bar);
      }
    }
    // (bounded waits; the outcome is made CTA-uniform before going on)
    ok = __syncthreads_and(mbar_wait(s_bar, it & 1, &abort_flag));
    if (!ok) break;
    tc_fence_after();
    // the S product has read Q buffer `buf`: refill it with tile it + 2
    if (warp == 0 && it + 2 < n_my) load_q(it + 2);
    float l = 0.f, score = 0.f;
    if (Lp <= 128) {
      // all of S in registers: one TMEM pass. Only the last 32-key chunk can
      // hold padding keys; they are set to -inf (their weights are 0).
      uint32_t sr[128];
      const int nc = Lp / 32;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (c < nc) tmem_ld32(tS + 32 * c, sr + 32 * c);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (c < nc) tmem_ld_wait32(sr + 32 * c);  // ties the loaded registers to the wait
#pragma unroll
      for (int j = 0; j < 128; ++j)
        if (j >= L) sr[j] = __float_as_uint(-INFINITY);
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c < nc) {
#pragma unroll
          for (int i = 0; i < 32; i += 8)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              m4[k] = fmax3(m4[k], __uint_as_float(sr[32 * c + i + 2 * k]), __uint_as_float(sr[32 * c + i + 2 * k + 1]));
        }
      }
      const float mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
      const uint64_t sl2x2 = f2_pack(sl2, sl2), neg2 = f2_pack(-mx * sl2, -mx * sl2);
      uint64_t lacc[2] = {0, 0}, sacc[2] = {0, 0};  // packed row sums and weighted sums
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c >= nc) continue;
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int j0 = 32 * c + 2 * i;
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[j0]), __uint_as_float(sr[j0 + 1])), sl2x2, neg2), x0, x1);
          const float a = ex2_approx(x0), bb = ex2_approx(x1);
          const uint64_t e2 = f2_pack(a, bb);
          const float2 w2 = *reinterpret_cast<const float2*>(sw + j0);
          lacc[i & 1] = f2_add(lacc[i & 1], e2);
          sacc[i & 1] = f2_fma(f2_pack(w2.x, w2.y), e2, sacc[i & 1]);
          pk[i] = pack_bf16x2(a, bb);
        }
        if (p.O != nullptr) tmem_st16(tS + 16 * c, pk);
      }
      float l0, l1, l2, l3, s0, s1, s2, s3;
      f2_unpack(lacc[0], l0, l1);
      f2_unpack(lacc[1], l2, l3);
      f2_unpack(sacc[0], s0, s1);
      f2_unpack(sacc[1], s2, s3);
      l = (l0 + l1) + (l2 + l3);
      score = (s0 + s1) + (s2 + s3);
    } else {
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
    }
    if (p.partial != nullptr && valid)
      p.partial[(static_cast<size_t>(b) * p.H + h) * p.nq + q_row] = score / l;

    if (p.O != nullptr) {
      // O = P Vy / l
      tmem_st_wait();
      tc_fence_before();
      __syncthreads();
      if (tid == 0 && !abort_flag) {
        tc_fence_after();
        for (int kk = 0; kk < Lp / 16; ++kk)
          umma_ts(tbase + s_region, tbase + kk * 8, make_sdesc(aV + kk * 16 * 64, Mp * 64, 512, kSwizzle64B), idPV,
                  kk > 0 ? 1u : 0u);
        umma_commit(o_bar);
      }
      ok = __syncthreads_and(mbar_wait(o_bar, it & 1, &abort_flag));
      if (!ok) break;
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
    // every thread has read S / O of this tile before the next S overwrites them
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (!ok && warp == 0) {
    // let the query loads this CTA started land before it exits
    for (int i = q_issued - 2 < 0 ? 0 : q_issued - 2; i < q_issued; ++i)
      mbar_wait_drain(&q_full[i & 1], (i >> 1) & 1);
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
