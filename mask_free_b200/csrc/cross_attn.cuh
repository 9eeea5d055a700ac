// cross_attn.cuh - image->text cross-attention with the text padding kept as
// per-sample valid key lengths (Eq. (4), Eq. (17)), and the per-head PCSP
// partial scores built from the same probabilities (Eq. (9), (10)).
//
// All M <= 256 text keys of a (b, h) fit one tile, so the softmax is exact in
// one pass over them. A CTA (one per SM) owns a range of 128-row query tiles
// of one (b, h) and pipelines them:
//   warp 0      TMA producer: query tiles (dense rows, or rows of S via
//               gather4) into a ring of QS shared-memory slots;
//   warps 1, 2  MMA issuers, one per softmax warpgroup (even / odd tiles;
//               the whole warp runs the loop, one elected lane issues):
//               S = Q Ky^T (N = Lp = ceil32(valid_len)) into TMEM, then
//               O = P Vy with P read from TMEM;
//   warp 3      output store: the bf16 O tile, staged by the warpgroup in
//               shared memory, leaves by TMA store;
//   warps 4..11 two softmax warpgroups, one query row per thread: max over
//               the keys, p = 2^(s*scale*log2(e) - max), l = sum p,
//               score = sum_j w_j p_j / l (the PCSP partial of this head),
//               P (bf16) into TMEM; after P V, O / l into the staging buffer.
// Before the first tile the text key / value rows [0, Lp) are copied into the
// swizzled layouts the tensor core reads, zeros for rows >= valid_len
// (padding rows are never read, so they may hold any bytes). The padding
// keys are masked by the tensor core itself: one more K = 16 step adds
// ones(128 x 16) . bias(Lp x 16)^T to S, with bias rows 0 for valid keys and
// -inf for padding keys, so S arrives with -inf in every padding column and
// the softmax has no mask to apply.
//
// Two TMEM layouts (512 columns; see cross_sep_p below): for D <= 96 and
// M <= 128, S0, S1, O0, O1 and one P buffer shared by the warpgroups in
// alternation, with S released as soon as it is loaded and the output
// staged in two buffers of its own; otherwise warpgroup g owns
// [256g, 256g + 256) (S at 0 with P over it, O at 128) and stages its output
// in the slot its query tile came from.
#pragma once

#include <type_traits>

#include "flash_attn.cuh"

namespace safe {

struct CrossParams {
  CUtensorMap q_map[2];   // 4-D dense Q map per chunk
  CUtensorMap qg_map[2];  // 2-D gather map per chunk
  CUtensorMap o_map[2];   // 4-D map of O [B, nq, H, D] per chunk (stores)
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
  int qs;  // query-tile slots in shared memory
};

constexpr int kCrossThreads = 384;
constexpr int kCrossMaxSmem = 232448 - 1024;  // dynamic shared memory limit of one CTA, less room for the static part
constexpr int kCrossMinSmem = 120 * 1024;  // keeps the CTA alone on its SM (it holds all of TMEM)

// Separate-P layout (D <= 96, M <= 128): TMEM S0 [0,128), S1 [128,256),
// O0 [256,256+D), O1 [256+D,256+2D), one 64-column P buffer [256+2D,+64)
// shared by the two warpgroups (P of tile i is written after P V of tile
// i-1). S is released as soon as it is loaded, so the next S of a warpgroup
// is computed while it exponentiates; the output is staged in two buffers of
// its own, so a query slot returns to the producer as soon as S is done.
// Otherwise P overwrites S, the warpgroup owns [256g, 256g+256) (S at 0, O at
// 128) and the output is staged in the slot its queries came from.
template <int D>
__host__ __device__ constexpr bool cross_sep_p(int M) {
  return D <= 96 && M <= 128;
}
template <int D>
__host__ __device__ constexpr int cross_smem_need(int M, int qs) {
  return 1024 + (qs + (cross_sep_p<D>(M) ? 2 : 0)) * TileCfg<D>::kTileBytes + 2 * (((M + 31) / 32) * 32) * D * 2 +
         128 * 32 + (((M + 31) / 32) * 32) * 32 + 256 * 4 + 256;
}
// Slots that fit next to the text keys / values (4 at most, 2 at least).
template <int D>
__host__ __device__ constexpr int cross_slots(int M) {
  return cross_smem_need<D>(M, 4) <= kCrossMaxSmem ? 4 : (cross_smem_need<D>(M, 3) <= kCrossMaxSmem ? 3 : 2);
}
template <int D>
__host__ __device__ constexpr int cross_smem_bytes(int M) {
  return cross_smem_need<D>(M, cross_slots<D>(M)) < kCrossMinSmem ? kCrossMinSmem
                                                                  : cross_smem_need<D>(M, cross_slots<D>(M));
}

// kO: O is written (cross-attention); otherwise only the PCSP partials
// (p.O == nullptr), and the softmax builds no P.
template <int D, bool kSep, bool kO>
__global__ void __launch_bounds__(kCrossThreads, 1) cross_attn_kernel(const __grid_constant__ CrossParams p) {
  using C = TileCfg<D>;
  constexpr int TB = C::kTileBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int QS = p.qs;
  const int Mp = ((p.M + 31) / 32) * 32;
  uint8_t* sQ = sm;  // QS query-tile slots (aliased layout: also the output staging)
  uint8_t* sOut = sQ + QS * TB;  // separate-P layout: two output staging buffers
  uint8_t* sKy = sOut + (kSep ? 2 * TB : 0);
  uint8_t* sVy = sKy + Mp * D * 2;
  uint8_t* sOnes = sVy + Mp * D * 2;  // 128 rows x 16 bf16 ones (32-byte rows)
  uint8_t* sBias = sOnes + 128 * 32;  // Mp rows x 16 bf16: 0 (valid key) or -inf
  float* sw = reinterpret_cast<float*>(sBias + Mp * 32);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sw + 256);
  uint64_t* q_full = bars;         // [4] per slot
  uint64_t* q_empty = bars + 4;    // [4]
  // [4] output tile written to its staging buffer (per buffer: a buffer's
  // next output waits for this one's store, so its phases are never skipped)
  uint64_t* o_staged = bars + 8;
  uint64_t* s_full = bars + 12;   // [2] per warpgroup
  uint64_t* s_free = bars + 14;   // [2] S loaded (separate-P layout)
  uint64_t* p_full = bars + 16;   // [2]
  uint64_t* pv_done = bars + 18;  // [2] P V complete: the P buffer is free (separate-P layout)
  uint64_t* o_full = bars + 20;   // [2]
  uint64_t* t_free = bars + 22;   // [2] the warpgroup's TMEM output (aliased: and S) read
  uint64_t* drained = bars + 24;  // [2] issuer's MMAs all complete
  uint64_t* out_free = bars + 26;  // [2] staging buffer read by its store (separate-P layout)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 28);
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.z, h = blockIdx.y;
  const int n_tiles = (p.nq + 127) / 128;
  const int per = (n_tiles + gridDim.x - 1) / gridDim.x;
  const int tile0 = blockIdx.x * per;
  const int tile1 = tile0 + per < n_tiles ? tile0 + per : n_tiles;
  if (tile0 >= tile1) return;  // uniform for the CTA, before any barrier or TMEM use
  const int n_my = tile1 - tile0;
  // (runtime for kO: the O-writing kernel compiles as it did with one
  // instantiation for both uses, which its register allocation prefers)
  const bool has_o = kO && p.O != nullptr;

  int L = __ldg(p.valid_len + b);
  if (L < 1 || L > p.M) {
    if (tid == 0) raise_status(1 << 5);
    L = L < 1 ? 1 : p.M;
  }
  const int Lp = ((L + 31) / 32) * 32;

  // TMEM columns of warpgroup g's S and O, and of P
  auto col_S = [](int g) -> uint32_t { return kSep ? 128u * g : 256u * g; };
  auto col_O = [](int g) -> uint32_t { return kSep ? 256u + static_cast<uint32_t>(D) * g : 256u * g + 128u; };
  auto col_P = [](int g) -> uint32_t { return kSep ? 256u + 2u * D : 256u * g; };

  if (tid == 0) {
    abort_flag = 0;
    for (int i = 0; i < 4; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&o_staged[i], 128);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(&s_full[g], 1);
      mbar_init(&s_free[g], 128);
      mbar_init(&p_full[g], 128);
      mbar_init(&pv_done[g], 1);
      mbar_init(&o_full[g], 1);
      mbar_init(&t_free[g], 128);
      mbar_init(&drained[g], 1);
      mbar_init(&out_free[g], 1);
    }
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  // query tile `it` of this CTA -> slot it % QS (issued by the whole warp 0)
  auto load_q = [&](int it) {
    const int slot = it % QS;
    uint8_t* dst = sQ + slot * TB;
    const int q0 = (tile0 + it) * 128;
    if (lane == 0) mbar_arrive_expect_tx(&q_full[slot], TB);
    __syncwarp();
    if (!p.gather) {
      if (lane == 0)
        for (int c = 0; c < C::kChunks; ++c) tma_load_4d(dst + C::chunk_off(c), &p.q_map[c], &q_full[slot], 64 * c, h, q0, b);
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
        tma_gather4(dst + C::chunk_off(c) + 4 * lane * C::row_bytes(c), &p.qg_map[c], &q_full[slot],
                    h * D + 64 * c, y[0], y[1], y[2], y[3]);
    }
  };
  int q_issued = 0;
  if (warp == 0) {
    for (; q_issued < n_my && q_issued < QS; ++q_issued) load_q(q_issued);
  } else if (warp >= 3) {
    // text keys / values -> swizzled shared memory (zeros past valid_len);
    // eight 16-byte units per thread are loaded before any is stored
    constexpr int kUnits = D / 8;  // 16-byte units per row
    constexpr int kCopyThreads = kCrossThreads - 96;
    const int ct = tid - 96;
    const size_t row_stride = static_cast<size_t>(p.H) * D;  // elements between text tokens
    const __nv_bfloat16* kbase = p.Ky + (static_cast<size_t>(b) * p.M * p.H + h) * D;
    const __nv_bfloat16* vbase = p.Vy + (static_cast<size_t>(b) * p.M * p.H + h) * D;
    const int total = Lp * kUnits;
    for (int e0 = ct; e0 < total; e0 += 8 * kCopyThreads) {
      uint4 kv[8], vv[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int e = e0 + k * kCopyThreads;
        const int r = e / kUnits, u = e % kUnits;
        kv[k] = make_uint4(0, 0, 0, 0);
        vv[k] = make_uint4(0, 0, 0, 0);
        if (e < total && r < L) {
          kv[k] = __ldg(reinterpret_cast<const uint4*>(kbase + r * row_stride) + u);
          if (has_o) vv[k] = __ldg(reinterpret_cast<const uint4*>(vbase + r * row_stride) + u);
        }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int e = e0 + k * kCopyThreads;
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
    // mask operands (rows are uniform, so the 32-byte swizzle leaves them as
    // they are)
    for (int e = ct; e < 128 * 2; e += kCopyThreads)
      reinterpret_cast<uint4*>(sOnes)[e] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    for (int e = ct; e < Lp * 2; e += kCopyThreads) {
      const uint32_t v = (e >> 1) < L ? 0u : 0xFF80FF80u;
      reinterpret_cast<uint4*>(sBias)[e] = make_uint4(v, v, v, v);
    }
    for (int j = ct; j < Lp; j += kCopyThreads) {
      float wj = 0.f;
      if (j < L) wj = p.w != nullptr ? __ldg(p.w + static_cast<size_t>(b) * p.M + j) : 1.f / static_cast<float>(L);
      sw[j] = wj;
    }
    fence_proxy_async_smem();
  }
  __syncthreads();

  if (warp < 4) {
  regs_dealloc<kRegsControl>();  // (warpgroup-wide, as is the increase below)
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    bool ok = true;
    for (; q_issued < n_my; ++q_issued) {
      const int slot = q_issued % QS;
      ok = warp_wait(&q_empty[slot], ((q_issued / QS) - 1) & 1, &abort_flag);
      if (!ok) break;
      load_q(q_issued);
    }
    if (lane == 0) {
      // the loads this CTA started have landed before it exits (already
      // true unless another role gave up)
      for (int i = q_issued - QS < 0 ? 0 : q_issued - QS; i < q_issued; ++i)
        mbar_wait_drain(&q_full[i % QS], (i / QS) & 1);
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    const int g = warp - 1;
    {
      // the whole warp runs the issue loop; the elected lane issues
      const uint32_t leader = elect_one_sync();
      const uint32_t tS = tbase + col_S(g), tO = tbase + col_O(g), tP = tbase + col_P(g);
      const uint32_t idS = make_idesc_bf16(128, Lp, 0, 0);
      constexpr uint32_t idPV = make_idesc_bf16(128, D, 0, 1);
      const uint32_t aK = smem_u32(sKy), aV = smem_u32(sVy);
      // S_i = Q_i Ky^T (+ the padding mask); the slot returns to the
      // producer once S_i is done unless the output is staged in it
      auto issue_S = [&](int i) {
        const uint32_t aQ = smem_u32(sQ + (i % QS) * TB);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int c = kk >> 2;
          const uint64_t bd = make_sdesc(aK + c * Mp * 128 + (kk & 3) * 32, 16, 8 * C::row_bytes(c), C::swizzle(c));
          umma_ss_if(leader, tS, kmajor_desc<D>(aQ, kk), bd, idS, kk > 0 ? 1u : 0u);
        }
        if (L < Lp)  // padding keys -> -inf
          umma_ss_if(leader, tS, make_sdesc(smem_u32(sOnes), 16, 256, kSwizzle32B),
                     make_sdesc(smem_u32(sBias), 16, 256, kSwizzle32B), idS, 1u);
        umma_commit_if(leader, &s_full[g]);
        if (kSep || !has_o) umma_commit_if(leader, &q_empty[i % QS]);
      };
      auto issue_PV = [&]() {
        for (int kk = 0; kk < Lp / 16; ++kk)
          umma_ts_if(leader, tO, tP + kk * 8, make_sdesc(aV + kk * 16 * 64, Mp * 64, 512, kSwizzle64B), idPV, kk > 0 ? 1u : 0u);
        if (kSep) umma_commit_if(leader, &pv_done[g]);
        umma_commit_if(leader, &o_full[g]);
      };
      if constexpr (kSep) {
        // per tile: the next S as soon as the softmax has loaded the
        // current one, then P V once P is written
        bool ok = g < n_my && warp_wait(&q_full[g % QS], (g / QS) & 1, &abort_flag);
        if (ok) {
          tc_fence_after();
          issue_S(g);
        }
        for (int i = g; ok && i < n_my; i += 2) {
          const int k = i >> 1;
          if (i + 2 < n_my) {
            ok = warp_wait(&q_full[(i + 2) % QS], ((i + 2) / QS) & 1, &abort_flag) &&
                 warp_wait(&s_free[g], k & 1, &abort_flag);
            if (!ok) break;
            tc_fence_after();
            issue_S(i + 2);
          }
          if (has_o) {
            ok = warp_wait(&p_full[g], k & 1, &abort_flag) && (k == 0 || warp_wait(&t_free[g], (k - 1) & 1, &abort_flag));
            if (!ok) break;
            tc_fence_after();
            issue_PV();
          }
        }
      } else {
        for (int i = g; i < n_my; i += 2) {
          const int k = i >> 1;
          if (!warp_wait(&q_full[i % QS], (i / QS) & 1, &abort_flag)) break;
          // the previous tile of this warpgroup has released S (and, when S
          // reaches into the O columns, its output)
          if (k > 0) {
            uint64_t* prev = (has_o && Lp <= 128) ? &o_full[g] : &t_free[g];
            if (!warp_wait(prev, (k - 1) & 1, &abort_flag)) break;
          }
          tc_fence_after();
          issue_S(i);
          if (!has_o) continue;
          if (!warp_wait(&p_full[g], k & 1, &abort_flag)) break;
          if (k > 0 && !warp_wait(&t_free[g], (k - 1) & 1, &abort_flag)) break;
          tc_fence_after();
          issue_PV();
        }
      }
      // every MMA the leader issued has completed before TMEM is released
      umma_commit_if(leader, &drained[g]);
      mbar_wait_drain(&drained[g], 0);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ output store
    if (has_o && lane == 0) {
      for (int i = 0; i < n_my; ++i) {
        const int buf = kSep ? (i & 1) : (i % QS);
        if (!mbar_wait(&o_staged[buf], kSep ? ((i >> 1) & 1) : ((i / QS) & 1), &abort_flag)) break;
        const uint8_t* src = kSep ? sOut + buf * TB : sQ + buf * TB;
        const int q0 = (tile0 + i) * 128;
        for (int c = 0; c < C::kChunks; ++c) tma_store_4d(&p.o_map[c], src + C::chunk_off(c), 64 * c, h, q0, b);
        bulk_commit_group();
        bulk_wait_read_all();
        mbar_arrive(kSep ? &out_free[buf] : &q_empty[buf]);
      }
      bulk_wait_all();
    }
  }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    regs_alloc<kRegsSoftmax>();
    const int g = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tbase + col_S(g) + lane_addr;
    const uint32_t tO = tbase + col_O(g) + lane_addr;
    const uint32_t tP = tbase + col_P(g) + lane_addr;
    const float sl2 = p.scale_log2;
    float linv_even = 1.f, linv_odd = 1.f;  // 1 / l of this warpgroup's last two tiles
    const bool want_score = p.partial != nullptr;

    // softmax of tile i: probabilities, l and the PCSP partial; P -> TMEM
    auto softmax = [&](int i) -> bool {
      const int k = i >> 1;
      const int q_row = (tile0 + i) * 128 + row;
      if (!warp_wait(&s_full[g], k & 1, &abort_flag)) return false;
      tc_fence_after();
      float l = 0.f, score = 0.f;
      // all of S in registers: one TMEM pass (padding keys hold -inf and
      // weight 0), specialised on the number NC of 32-key chunks so that
      // every register index is static, and on whether the weighted sum of
      // the PCSP partial is wanted (SC)
      auto one_pass = [&](auto nc_tag, auto sc_tag) -> bool {
        constexpr int NC = decltype(nc_tag)::value;
        constexpr bool SC = decltype(sc_tag)::value;
        uint32_t sr[32 * NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_ld32(tS + 32 * c, sr + 32 * c);
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_ld_wait32(sr + 32 * c);  // ties the loaded registers to the wait
        if (kSep || !has_o) {
          tc_fence_before();
          mbar_arrive(kSep ? &s_free[g] : &t_free[g]);  // S may be overwritten
        }
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < 32 * NC; j += 8)
#pragma unroll
          for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], __uint_as_float(sr[j + 2 * q]), __uint_as_float(sr[j + 2 * q + 1]));
        const float mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
        const uint64_t sl2x2 = f2_pack(sl2, sl2), neg2 = f2_pack(-mx * sl2, -mx * sl2);
        uint64_t lacc[2] = {0, 0}, sacc[2] = {0, 0};  // packed row sums and weighted sums
        uint32_t pk[16 * NC];
#pragma unroll
        for (int i2 = 0; i2 < 16 * NC; ++i2) {
          const int j0 = 2 * i2;
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[j0]), __uint_as_float(sr[j0 + 1])), sl2x2, neg2), x0, x1);
          const float a = ex2_approx(x0), bb = ex2_approx(x1);
          const uint64_t e2 = f2_pack(a, bb);
          lacc[i2 & 1] = f2_add(lacc[i2 & 1], e2);
          if constexpr (SC) {
            const float2 w2 = *reinterpret_cast<const float2*>(sw + j0);
            sacc[i2 & 1] = f2_fma(f2_pack(w2.x, w2.y), e2, sacc[i2 & 1]);
          }
          pk[i2] = pack_bf16x2(a, bb);
          if (!kSep && has_o && (i2 & 15) == 15) tmem_st16(tP + (i2 - 15), pk + (i2 - 15));
        }
        if (kSep && has_o) {
          // the shared P buffer: tile i-1's P V (the other warpgroup) has
          // read it
          if (i > 0 && !warp_wait(&pv_done[g ^ 1], ((i - 1) >> 1) & 1, &abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < NC; ++c) tmem_st16(tP + 16 * c, pk + 16 * c);
        }
        float l0, l1, l2, l3, s0, s1, s2, s3;
        f2_unpack(lacc[0], l0, l1);
        f2_unpack(lacc[1], l2, l3);
        f2_unpack(sacc[0], s0, s1);
        f2_unpack(sacc[1], s2, s3);
        l = (l0 + l1) + (l2 + l3);
        score = (s0 + s1) + (s2 + s3);
        return true;
      };
      if (Lp <= 128) {
        bool ok;
        const std::true_type sc_on;
        const std::false_type sc_off;
        switch (Lp / 32) {
          case 1: ok = want_score ? one_pass(std::integral_constant<int, 1>{}, sc_on)
                                  : one_pass(std::integral_constant<int, 1>{}, sc_off); break;
          case 2: ok = want_score ? one_pass(std::integral_constant<int, 2>{}, sc_on)
                                  : one_pass(std::integral_constant<int, 2>{}, sc_off); break;
          case 3: ok = want_score ? one_pass(std::integral_constant<int, 3>{}, sc_on)
                                  : one_pass(std::integral_constant<int, 3>{}, sc_off); break;
          default: ok = want_score ? one_pass(std::integral_constant<int, 4>{}, sc_on)
                                   : one_pass(std::integral_constant<int, 4>{}, sc_off); break;
        }
        if (!ok) return false;
      } else {
        // (aliased layout only) two passes over S, 32 keys at a time,
        // specialised on the number NC of chunks: pass 1 the row max, pass 2
        // the probabilities, the sums and P (P chunk c lands on S columns
        // already read). The padding columns hold -inf from the mask step of
        // the S product and weight 0, so no key needs a test.
        auto two_pass = [&](auto nc_tag, auto sc_tag) {
          constexpr int NC = decltype(nc_tag)::value;
          constexpr bool SC = decltype(sc_tag)::value;
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            uint32_t sr[32];
            tmem_ld32(tS + 32 * c, sr);
            tmem_ld_wait32(sr);
#pragma unroll
            for (int j = 0; j < 32; j += 8)
#pragma unroll
              for (int q = 0; q < 4; ++q)
                m4[q] = fmax3(m4[q], __uint_as_float(sr[j + 2 * q]), __uint_as_float(sr[j + 2 * q + 1]));
          }
          const float mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
          const uint64_t sl2x2 = f2_pack(sl2, sl2), neg2 = f2_pack(-mx * sl2, -mx * sl2);
          uint64_t lacc[2] = {0, 0}, sacc[2] = {0, 0};  // packed row sums and weighted sums
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            uint32_t sr[32];
            tmem_ld32(tS + 32 * c, sr);
            tmem_ld_wait32(sr);
            uint32_t pk[16];
#pragma unroll
            for (int i2 = 0; i2 < 16; ++i2) {
              const int j0 = 32 * c + 2 * i2;
              float x0, x1;
              f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * i2]), __uint_as_float(sr[2 * i2 + 1])), sl2x2, neg2),
                        x0, x1);
              const float a = ex2_approx(x0), bb = ex2_approx(x1);
              const uint64_t e2 = f2_pack(a, bb);
              lacc[i2 & 1] = f2_add(lacc[i2 & 1], e2);
              if constexpr (SC) {
                const float2 w2 = *reinterpret_cast<const float2*>(sw + j0);
                sacc[i2 & 1] = f2_fma(f2_pack(w2.x, w2.y), e2, sacc[i2 & 1]);
              }
              pk[i2] = pack_bf16x2(a, bb);
            }
            if (has_o) tmem_st16(tP + 16 * c, pk);
          }
          float l0, l1, l2, l3, s0, s1, s2, s3;
          f2_unpack(lacc[0], l0, l1);
          f2_unpack(lacc[1], l2, l3);
          f2_unpack(sacc[0], s0, s1);
          f2_unpack(sacc[1], s2, s3);
          l = (l0 + l1) + (l2 + l3);
          score = (s0 + s1) + (s2 + s3);
        };
        const std::true_type sc_on;
        const std::false_type sc_off;
        switch (Lp / 32) {
          case 5: want_score ? two_pass(std::integral_constant<int, 5>{}, sc_on)
                             : two_pass(std::integral_constant<int, 5>{}, sc_off); break;
          case 6: want_score ? two_pass(std::integral_constant<int, 6>{}, sc_on)
                             : two_pass(std::integral_constant<int, 6>{}, sc_off); break;
          case 7: want_score ? two_pass(std::integral_constant<int, 7>{}, sc_on)
                             : two_pass(std::integral_constant<int, 7>{}, sc_off); break;
          default: want_score ? two_pass(std::integral_constant<int, 8>{}, sc_on)
                              : two_pass(std::integral_constant<int, 8>{}, sc_off); break;
        }
        if (!has_o) {
          tc_fence_before();
          mbar_arrive(&t_free[g]);
        }
      }
      if (has_o) {
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[g]);
      }
      if (p.partial != nullptr && q_row < p.nq) p.partial[(static_cast<size_t>(b) * p.H + h) * p.nq + q_row] = score / l;
      if (k & 1) linv_odd = 1.f / l;
      else linv_even = 1.f / l;
      return true;
    };

    // O = P Vy / l of tile i -> bf16 into a staging buffer laid out like a
    // query tile for the store: the warpgroup's own (separate-P layout) or
    // the slot of the tile's queries, which the S product has read
    auto epilogue = [&](int i) -> bool {
      const int k = i >> 1;
      if (!warp_wait(&o_full[g], k & 1, &abort_flag)) return false;
      if (kSep && k > 0 && !warp_wait(&out_free[g], (k - 1) & 1, &abort_flag)) return false;
      tc_fence_after();
      const float inv_l = (k & 1) ? linv_odd : linv_even;
      uint8_t* slot = kSep ? sOut + g * TB : sQ + (i % QS) * TB;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_ld_wait32(o);
        if (c == D / 32 - 1) {
          tc_fence_before();
          mbar_arrive(&t_free[g]);
        }
        uint32_t pk[16];
#pragma unroll
        for (int i2 = 0; i2 < 16; ++i2)
          pk[i2] = pack_bf16x2(__uint_as_float(o[2 * i2]) * inv_l, __uint_as_float(o[2 * i2 + 1]) * inv_l);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int u = 4 * c + v;  // 16-byte unit of the row
          const int cq = u >> 3, uc = u & 7;
          const int rb = C::row_bytes(cq);
          const int xr = (rb == 128) ? (row & 7) : ((row >> 1) & 3);
          *reinterpret_cast<uint4*>(slot + C::chunk_off(cq) + row * rb + ((uc ^ xr) << 4)) =
              make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&o_staged[kSep ? g : i % QS]);
      return true;
    };

    if constexpr (kSep) {
      // softmax of the next tile before the output of the previous one: its
      // P V has long finished by then
      for (int i = g;; i += 2) {
        if (i < n_my && !softmax(i)) break;
        if (has_o && i >= 2 && i - 2 < n_my && !epilogue(i - 2)) break;
        if (i >= n_my) break;
      }
    } else {
      for (int i = g; i < n_my; i += 2) {
        if (!softmax(i)) break;
        if (has_o && !epilogue(i)) break;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

// scores[b, i] (+)= (1/H) * sum_h partial[b, h, i], heads summed in order.
__global__ void pcsp_reduce_kernel(const float* __restrict__ partial, float* __restrict__ scores, int B, int H, int N,
                                   int accumulate) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int b = blockIdx.y;
  if (i >= N) return;
  // eight heads' loads in flight at a time, summed in head order
  const float* src = partial + static_cast<size_t>(b) * H * N + i;
  float acc = 0.f;
  for (int h0 = 0; h0 < H; h0 += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = h0 + u < H ? __ldg(src + static_cast<size_t>(h0 + u) * N) : 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (h0 + u < H) acc += v[u];
  }
  acc = acc / static_cast<float>(H);
  float* dst = scores + static_cast<size_t>(b) * N + i;
  *dst = accumulate ? *dst + acc : acc;
}

}  // namespace safe
