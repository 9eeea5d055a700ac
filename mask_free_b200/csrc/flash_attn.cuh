// flash_attn.cuh - mask-free attention over all N keys on tcgen05 tensor cores.
//
// Serves two calls of the SAFE-DiT hot path:
//   * dense image self-attention with the redundant mask elided (Eq. (3), (8)),
//   * SRSU selective self-attention (Eq. (16)): the query rows are the
//     sensitive set S, gathered from Q with TMA gather4, attending to all N
//     keys of the global K/V assembled from current and cached rows.
//
// One CTA owns two 128-row query tiles of one (b, h) and streams the key /
// value tiles of that head through a shared-memory ring:
//   warp 0       TMA producer (Q tiles once, then K_j / V_j per stage)
//   warp 1       MMA issuer (one thread): S_t = Q_t K_j^T into TMEM, then
//                O_t += P_t V_j with P_t read from TMEM (TS form)
//   warps 2..5   softmax for tile 0, warps 6..9 softmax for tile 1: each
//                thread owns one query row (one TMEM lane), reads S_t, keeps
//                the running max / sum in registers, writes P_t (bf16) back
//                into TMEM over S_t, rescales O_t lazily, and finally writes
//                O = O_t / l (bf16) and the log-sum-exp.
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256, 256+D), O1 [256+D, 256+2D).
// Online softmax in base 2: p = 2^(s*scale*log2(e) - m); O is only rescaled
// when the running max grows by more than 8 (p stays below 2^8 otherwise).
#pragma once

#include "sm100.cuh"

namespace safe {

template <int D>
struct TileCfg {
  static_assert(D == 64 || D == 96 || D == 128, "head dim");
  static constexpr int kChunks = (D + 63) / 64;
  static constexpr int kTileBytes = 128 * D * 2;  // 128 rows of D bf16
  static constexpr int kStages = D <= 64 ? 4 : (D <= 96 ? 3 : 2);
  // chunk c holds columns [64c, 64c + width(c)); 64-wide chunks use the 128B
  // swizzle (128-byte rows), the 32-wide tail of D = 96 the 64B swizzle.
  __host__ __device__ static constexpr int width(int c) { return (D - 64 * c) >= 64 ? 64 : (D - 64 * c); }
  __host__ __device__ static constexpr int row_bytes(int c) { return width(c) * 2; }
  __host__ __device__ static constexpr uint32_t chunk_off(int c) { return static_cast<uint32_t>(c) * 128u * 128u; }
  __host__ __device__ static constexpr uint32_t swizzle(int c) { return width(c) == 64 ? kSwizzle128B : kSwizzle64B; }
};

// K-major operand (rows of a 128-row tile, contiguous along the head dim):
// descriptor for the 16-element k-step kk.
template <int D>
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int kk) {
  using C = TileCfg<D>;
  const int c = kk >> 2;
  return make_sdesc(tile + C::chunk_off(c) + static_cast<uint32_t>(kk & 3) * 32u, 16, 8 * C::row_bytes(c),
                    C::swizzle(c));
}

// MN-major B operand (V tile: rows = keys, contiguous along the head dim):
// descriptor of chunk c for the 16-key step kk.
template <int D>
__device__ __forceinline__ uint64_t vmajor_desc(uint32_t tile, int c, int kk) {
  using C = TileCfg<D>;
  return make_sdesc(tile + C::chunk_off(c) + static_cast<uint32_t>(kk * 16 * C::row_bytes(c)), C::chunk_off(1),
                    8 * C::row_bytes(c), C::swizzle(c));
}

struct FlashParams {
  CUtensorMap q_map[2];   // 4-D [B, rows, H, D] map per chunk (dense / compact Q)
  CUtensorMap qg_map[2];  // 2-D [B*N, H*D] gather map per chunk (rows of S)
  CUtensorMap k_map[2];   // 4-D [B, N, H, D]
  CUtensorMap v_map[2];
  const int32_t* S;       // [B, n_q] query rows when gathering, else null
  __nv_bfloat16* O;       // [B, n_q, H, D]
  float* lse;             // [B, H, n_q] or null
  int B, N, H, n_q;
  float scale_log2;       // logit scale * log2(e)
  int gather;
};

constexpr int kFlashThreads = 320;

template <int D>
__host__ __device__ constexpr int flash_smem_bytes() {
  using C = TileCfg<D>;
  return 1024 /*align slack*/ + (2 + 2 * C::kStages) * C::kTileBytes + 256 /*barriers + tmem slot*/;
}

__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) return false;
  }
  return true;
}

template <int D>
__global__ void __launch_bounds__(kFlashThreads, 1) flash_fwd_kernel(const __grid_constant__ FlashParams p) {
  using C = TileCfg<D>;
  constexpr int ST = C::kStages;
  constexpr int TB = C::kTileBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = sm;
  uint8_t* sK = sQ + 2 * TB;
  uint8_t* sV = sK + ST * TB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + ST * TB);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* v_full = k_full + ST;
  uint64_t* kv_empty = v_full + ST;
  uint64_t* s_full = kv_empty + ST;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* drain = o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.z, h = blockIdx.y;
  const int q_base = blockIdx.x * 256;
  const int n_kv = (p.N + 127) / 128;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_full[t], 1);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int c = 0; c < C::kChunks; ++c) {
        tma_prefetch_desc(&p.k_map[c]);
        tma_prefetch_desc(&p.v_map[c]);
      }
      mbar_arrive_expect_tx(q_full, 2 * TB);
    }
    __syncwarp();
    if (!p.gather) {
      if (lane == 0) {
        for (int t = 0; t < 2; ++t)
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(sQ + t * TB + C::chunk_off(c), &p.q_map[c], q_full, 64 * c, h, q_base + t * 128, b);
      }
    } else {
      // lane l gathers rows 4l..4l+3 of each tile (indices clamped to the
      // last valid row for the ragged tail; out-of-range indices flagged)
      for (int t = 0; t < 2; ++t) {
        int y[4];
        for (int u = 0; u < 4; ++u) {
          int r = q_base + t * 128 + 4 * lane + u;
          r = r < p.n_q ? r : p.n_q - 1;
          int idx = __ldg(p.S + static_cast<size_t>(b) * p.n_q + r);
          if (idx < 0 || idx >= p.N) {
            raise_status(1 << 5);
            idx = 0;
          }
          y[u] = b * p.N + idx;
        }
        for (int c = 0; c < C::kChunks; ++c)
          tma_gather4(sQ + t * TB + C::chunk_off(c) + 4 * lane * C::row_bytes(c), &p.qg_map[c], q_full,
                      h * D + 64 * c, y[0], y[1], y[2], y[3]);
      }
    }
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % ST;
        if (j >= ST && !mbar_wait(&kv_empty[s], ((j / ST) - 1) & 1, &abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&k_full[s], TB);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(sK + s * TB + C::chunk_off(c), &p.k_map[c], &k_full[s], 64 * c, h, j * 128, b);
        mbar_arrive_expect_tx(&v_full[s], TB);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(sV + s * TB + C::chunk_off(c), &p.v_map[c], &v_full[s], 64 * c, h, j * 128, b);
        issued = j + 1;
      }
      if (!ok || abort_flag) {
        // let every copy this CTA started land before the CTA exits
        mbar_wait_drain(q_full, 0);
        for (int j = issued - ST < 0 ? 0 : issued - ST; j < issued; ++j) {
          mbar_wait_drain(&k_full[j % ST], (j / ST) & 1);
          mbar_wait_drain(&v_full[j % ST], (j / ST) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = make_idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idPV0 = make_idesc_bf16(128, C::width(0), 0, 1);
      constexpr uint32_t idPV1 = make_idesc_bf16(128, C::kChunks > 1 ? C::width(1) : 64, 0, 1);
      const uint32_t tS[2] = {tbase, tbase + 128};
      const uint32_t tO[2] = {tbase + 256, tbase + 256 + D};
      const uint32_t aQ[2] = {smem_u32(sQ), smem_u32(sQ + TB)};
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
      auto issue_S = [&](int t, int s) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(tS[t], kmajor_desc<D>(aQ[t], kk), kmajor_desc<D>(aK + s * TB, kk), idS, kk > 0 ? 1u : 0u);
      };
      auto issue_PV = [&](int t, int s, int j) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
          umma_ts(tO[t], tS[t] + kk * 8, vmajor_desc<D>(aV + s * TB, 0, kk), idPV0, acc);
          if (C::kChunks > 1)
            umma_ts(tO[t] + 64, tS[t] + kk * 8, vmajor_desc<D>(aV + s * TB, 1, kk), idPV1, acc);
        }
      };
      bool ok = mbar_wait(q_full, 0, &abort_flag) && mbar_wait(&k_full[0], 0, &abort_flag);
      if (ok) {
        tc_fence_after();
        issue_S(0, 0);
        umma_commit(&s_full[0]);
        issue_S(1, 0);
        umma_commit(&s_full[1]);
        for (int j = 0; j < n_kv && ok; ++j) {
          const int s = j % ST;
          ok = mbar_wait(&v_full[s], (j / ST) & 1, &abort_flag);
          for (int t = 0; t < 2 && ok; ++t) {
            ok = mbar_wait(&p_full[t], j & 1, &abort_flag);
            if (!ok) break;
            tc_fence_after();
            issue_PV(t, s, j);
            if (j + 1 < n_kv) {
              const int s1 = (j + 1) % ST;
              if (t == 0) {
                ok = mbar_wait(&k_full[s1], ((j + 1) / ST) & 1, &abort_flag);
                if (!ok) break;
                tc_fence_after();
              }
              issue_S(t, s1);
              umma_commit(&s_full[t]);
            } else {
              umma_commit(&o_full[t]);
            }
          }
          if (ok) umma_commit(&kv_empty[s]);
        }
      }
      if (!ok) {
        // wait for every MMA this thread issued before TMEM is released
        umma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tbase + lane_addr + t * 128;
    const uint32_t tO = tbase + lane_addr + 256 + t * D;
    const int q_row = q_base + t * 128 + row;
    const float sl2 = p.scale_log2;
    const int tail = p.N - (n_kv - 1) * 128;  // valid keys in the last tile
    float m_use = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      // every lane waits; the outcome is made warp-uniform before the
      // warp-collective tcgen05.ld below
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[t], j & 1, &abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld32(tS + 0, sr);
      tmem_ld32(tS + 32, sr + 32);
      tmem_ld32(tS + 64, sr + 64);
      tmem_ld32(tS + 96, sr + 96);
      tmem_ld_wait32(sr);
      tmem_ld_wait32(sr + 32);
      tmem_ld_wait32(sr + 64);
      tmem_ld_wait32(sr + 96);
      if (j == n_kv - 1 && tail < 128) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= tail) sr[c] = __float_as_uint(-INFINITY);
      }
      float mx0 = __uint_as_float(sr[0]), mx1 = __uint_as_float(sr[1]);
      float mx2 = __uint_as_float(sr[2]), mx3 = __uint_as_float(sr[3]);
#pragma unroll
      for (int c = 4; c < 128; c += 4) {
        mx0 = fmaxf(mx0, __uint_as_float(sr[c]));
        mx1 = fmaxf(mx1, __uint_as_float(sr[c + 1]));
        mx2 = fmaxf(mx2, __uint_as_float(sr[c + 2]));
        mx3 = fmaxf(mx3, __uint_as_float(sr[c + 3]));
      }
      const float m_cand = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
      float alpha = 1.f;
      bool need = false;
      if (j == 0) {
        m_use = m_cand;
      } else {
        need = m_cand > m_use + 8.f;
        if (need) {
          alpha = ex2_approx(m_use - m_cand);
          m_use = m_cand;
        }
      }
      const float neg = -m_use;
      float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float a = ex2_approx(fmaf(__uint_as_float(sr[32 * c + 2 * i]), sl2, neg));
          const float bb = ex2_approx(fmaf(__uint_as_float(sr[32 * c + 2 * i + 1]), sl2, neg));
          sum0 += a;
          sum1 += bb;
          pk[i] = pack_bf16x2(a, bb);
        }
        tmem_st16(tS + 16 * c, pk);
      }
      // O_t is idle here (PV_t of the previous step completed before S_t of
      // this step was committed), so the rescale can follow the P store.
      if (__any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
          tmem_ld_wait32(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + 32 * c, o);
        }
      }
      l = l * alpha + (sum0 + sum1);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(&o_full[t], 0, &abort_flag))) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool valid = q_row < p.n_q;
      __nv_bfloat16* orow = p.O + ((static_cast<size_t>(b) * p.n_q + (valid ? q_row : 0)) * p.H + h) * D;
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
      if (valid && p.lse != nullptr)
        p.lse[(static_cast<size_t>(b) * p.H + h) * p.n_q + q_row] = (m_use + __log2f(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, 512);
}

}  // namespace safe
