// linear.cuh - row-wise layers of the row-selective block on tcgen05 tensor cores.
//
// The row-selective block B^S of SAFE-DiT (Eq. (15)) evaluates its
// projections and MLP only on the sensitive rows; with the row selection P_S
// of Eq. (13) each such layer is
//     Y[b, r, :] = act( X[b, S[b, r], :] W^T + bias )
// (no S: every row in order, the dense block of Eq. (18)).
//
// Two kernels share the epilogue below: linear_pair_kernel (CTA pairs,
// 256 x 256 tiles; every row in order, which the entry point also uses for
// the rows of S once it has copied them into a compact matrix) and
// linear_kernel (one SM per 128 x 256 tile; it gathers the rows of S
// itself when there is no workspace for the copy).
//
// linear_kernel is persistent: one CTA per SM walks the 128 x 256 output tiles
// t = blockIdx.x, blockIdx.x + gridDim.x, ... (the column tile fastest, so
// CTAs running at the same time share their gathered rows of X through L2).
//   warp 0     producer: per 64-wide K chunk, the 128 rows of X (rows of
//              S: TMA gather4, lane l copies rows 4l .. 4l + 3; every row:
//              one tiled copy) and the 256 x 64 tile of W by one tiled copy,
//              both K-major with the 128B swizzle, into a 4-stage ring
//   warp 1     MMA issuer (the whole warp runs the loop, one elected lane
//              issues): tcgen05.mma M = 128, N = 256, K = 16 into one of
//              two 256-column TMEM accumulators (tile i uses buffer i & 1)
//   warp 2     TMEM allocation
//   warps 4..11 epilogue: tcgen05.ld of the accumulator (TMEM lane = row of
//              the tile; warps 4..7 columns 0..127, warps 8..11 columns
//              128..255), + bias, activation, bf16 rows to global memory;
//              the buffer is released once read, so the next tile's MMAs
//              overlap this tile's stores
// Every wait is bounded (sm100.cuh); a row index outside [0, N) is flagged
// and replaced by row 0.
#pragma once

#include "sm100.cuh"

namespace safe {

// ---------------------------------------------------------------- CTA pairs (cta_group::2)
// Rank of this CTA in its cluster.
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of shared-memory location `p` in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// Every thread of both CTAs of the cluster arrives and waits.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on an mbarrier given by its shared::cluster address (any CTA of the cluster).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t caddr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}
// TMEM of a CTA pair: one warp of each CTA of the pair (the same warp index
// in both) allocates and frees, with the same destination slot.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Pair MMA, issued by the even CTA: D (M = 256: rows 0..127 in the even CTA's
// TMEM, 128..255 in the odd one's) (+)= A B^T, A's rows and B's rows (the
// N columns) split in halves between the two CTAs' shared memory at the
// same offsets as the descriptors give.
__device__ __forceinline__ void umma_pair_ss_if(uint32_t leader, uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 e, %5, 0;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(leader)
      : "memory");
}
// Arrive on the mbarrier at shared::cluster address `caddr` (either CTA of
// the pair) once the pair MMAs this thread issued so far have completed.
__device__ __forceinline__ void umma_pair_commit_if(uint32_t leader, uint32_t caddr) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "setp.ne.b32 e, %1, 0;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(caddr),
      "r"(leader)
      : "memory");
}
// 2-D tiled TMA load into this CTA's shared memory whose completion is
// counted on the mbarrier at shared::cluster address `mbar` (the pair's
// even CTA), box set by the tensor map.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t mbar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(mbar), "r"(c0), "r"(c1)
      : "memory");
}

struct LinearParams {
  CUtensorMap x_map;    // 2-D [B*N, d_in], box 64 x 1 (gather4)
  CUtensorMap xt_map;   // 2-D [B*N, d_in], box 64 x 128 (every row: one tiled copy)
  CUtensorMap w_map;    // 2-D [d_out, d_in], box 64 x 256
  CUtensorMap w2_map;   // 2-D [d_out, d_in], box 64 x 128 (a CTA's half of a pair's 256 columns)
  const int32_t* S;     // [B, R] rows of X, or null (rows 0 .. R-1)
  const float* bias;    // [d_out] or null
  __nv_bfloat16* Y;     // [B, R, d_out]
  int B, N, R, d_in, d_out, act;
  int m_tiles;          // row tiles per sample: ceil(R / 128)
  int n_tiles;          // column tiles: ceil(d_out / 256)
  int tiles;            // B * m_tiles * n_tiles
};

constexpr int kLinThreads = 384;  // warps 0-3 producer / MMA / TMEM, warps 4-11 epilogue
constexpr int kLinStages = 4;
constexpr int kLinABytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kLinBBytes = 256 * 128;  // 256 rows x 64 bf16
constexpr int kLinSmem = 1024 + kLinStages * (kLinABytes + kLinBBytes) + 256;

// GELU, tanh form (Hendrycks and Gimpel): 0.5 x (1 + tanh(u)) with
// u = sqrt(2/pi) (x + 0.044715 x^3), evaluated through the identity
// 0.5 (1 + tanh(u)) = 1 / (1 + e^(-2u)): one exponential on the exp unit and
// one division, with no cancellation where tanh(u) approaches -1 (the
// quotient tends to -0 for very negative x).
__device__ __forceinline__ float gelu_tanh_f(float x) {
  const float u = 0.7978845608028654f * fmaf(0.044715f * x, x * x, x);
  return __fdividef(x, 1.f + ex2_approx(-2.8853900817779268f * u));  // e^(-2u) = 2^(-2u log2(e))
}

// Xg[b, r, :] = X[b, S[b, r], :] for r < k, one warp per row, 16-byte
// units (d_in is a multiple of 8). An index outside [0, N) is flagged and
// row 0 is copied instead, as the gathering GEMM does.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ X, const int32_t* __restrict__ S,
                                                          uint4* __restrict__ Xg, int B, int N, int k,
                                                          int units_per_row) {
  pdl_launch_dependents();  // a dependent attention kernel may set up meanwhile
  const int lane = threadIdx.x & 31;
  const long long w = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (w >= static_cast<long long>(B) * k) return;
  const int b = static_cast<int>(w / k), r = static_cast<int>(w % k);
  int idx = __ldg(S + static_cast<size_t>(b) * k + r);
  if (idx < 0 || idx >= N) {
    if (lane == 0) raise_status(1 << 5);
    idx = 0;
  }
  const uint4* src = X + (static_cast<size_t>(b) * N + idx) * units_per_row;
  uint4* dst = Xg + (static_cast<size_t>(b) * k + r) * units_per_row;
  for (int u = lane; u < units_per_row; u += 32) dst[u] = __ldg(src + u);
}

// Epilogue of one output tile, run by eight warps: warp 4 + 4e + q reads
// TMEM lanes 32q .. 32q + 31 (rows of the tile) and columns
// [128e, 128e + 128) of the accumulator at `tacc` (four 32-column chunks),
// adds the bias, applies the activation and stores bf16 into `yrow` (the
// tile row's output, columns from n0). `release` is called once this
// thread's last chunk is in registers (the accumulator may then be reused).
template <typename Release>
__device__ __forceinline__ void linear_epilogue_tile(const LinearParams& p, uint32_t tacc, int e, int n0,
                                                     __nv_bfloat16* yrow, bool valid, Release release) {
  const bool bias_vec = (reinterpret_cast<uintptr_t>(p.bias) & 15u) == 0;
#pragma unroll 1
  for (int c = 4 * e; c < 4 * e + 4; ++c) {
    uint32_t v[32];
    tmem_ld32(tacc + 32 * c, v);
    tmem_ld_wait32(v);
    if (c == 4 * e + 3) {
      tc_fence_before();
      release();
    }
    const int nc = n0 + 32 * c;
    if (nc >= p.d_out) continue;
    // the chunk's 32 bias values: 8 vector loads (the same for every row,
    // so they come from L1), or element by element at the ragged last chunk
    // or a bias that is not 16-byte aligned
    float bv[32];
    if (p.bias == nullptr) {
#pragma unroll
      for (int k = 0; k < 32; ++k) bv[k] = 0.f;
    } else if (bias_vec && nc + 32 <= p.d_out) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 b4 = __ldg(reinterpret_cast<const float4*>(p.bias + nc) + u);
        bv[4 * u] = b4.x;
        bv[4 * u + 1] = b4.y;
        bv[4 * u + 2] = b4.z;
        bv[4 * u + 3] = b4.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < 32; ++k) bv[k] = nc + k < p.d_out ? __ldg(p.bias + nc + k) : 0.f;
    }
    uint32_t pk[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      float f0 = __uint_as_float(v[2 * k]) + bv[2 * k], f1 = __uint_as_float(v[2 * k + 1]) + bv[2 * k + 1];
      if (p.act == 1) {
        f0 = gelu_tanh_f(f0);
        f1 = gelu_tanh_f(f1);
      }
      pk[k] = pack_bf16x2(f0, f1);
    }
    if (valid) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (nc + 8 * u < p.d_out)
          *reinterpret_cast<uint4*>(yrow + nc + 8 * u) = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2],
                                                                    pk[4 * u + 3]);
    }
  }
}

__global__ void __launch_bounds__(kLinThreads, 1) linear_kernel(const __grid_constant__ LinearParams p) {
  constexpr int ST = kLinStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = sm;
  uint8_t* sB = sA + ST * kLinABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + ST * kLinBBytes);  // [ST] stage loaded
  uint64_t* empty = full + ST;                                          // [ST] stage consumed
  uint64_t* acc_full = empty + ST;                                      // [2] accumulator complete
  uint64_t* acc_empty = acc_full + 2;                                   // [2] accumulator read back
  uint64_t* drain = acc_empty + 2;                                      // MMA abort path
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = (p.d_in + 63) / 64;
  // tiles of this CTA: t = blockIdx.x + i * gridDim.x
  const int n_local = p.tiles > static_cast<int>(blockIdx.x)
                          ? (p.tiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                          : 0;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 256);  // every epilogue thread
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 2) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  auto tile_coords = [&](int i, int& b, int& r0, int& n0) {
    const int t = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    const int nt = t % p.n_tiles, mt = t / p.n_tiles;
    b = mt / p.m_tiles;
    r0 = (mt % p.m_tiles) * 128;
    n0 = nt * 256;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(p.S != nullptr ? &p.x_map : &p.xt_map);
      tma_prefetch_desc(&p.w_map);
    }
    int issued = 0;  // k chunks issued over all tiles
    bool ok = true;
    for (int i = 0; i < n_local && ok; ++i) {
      int b, r0, n0;
      tile_coords(i, b, r0, n0);
      // rows 4 lane .. 4 lane + 3 of the tile (the ragged tail repeats the
      // last row; its outputs are not stored)
      int y[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        int r = r0 + 4 * lane + u;
        r = r < p.R ? r : p.R - 1;
        int idx = p.S != nullptr ? __ldg(p.S + static_cast<size_t>(b) * p.R + r) : r;
        if (idx < 0 || idx >= p.N) {
          raise_status(1 << 5);
          idx = 0;
        }
        y[u] = b * p.N + idx;
      }
      for (int kc = 0; kc < nk; ++kc) {
        const int g = i * nk + kc, s = g % ST;
        if (g >= ST && !warp_wait(&empty[s], ((g / ST) - 1) & 1, &abort_flag)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], kLinABytes + kLinBBytes);
          tma_load_2d(sB + s * kLinBBytes, &p.w_map, &full[s], 64 * kc, n0);
          // every row: rows r0 .. r0 + 127 of sample b in one copy (rows
          // past the sample's end are other samples' rows or the zero fill
          // past the tensor; their outputs are not stored)
          if (p.S == nullptr) tma_load_2d(sA + s * kLinABytes, &p.xt_map, &full[s], 64 * kc, b * p.N + r0);
        }
        __syncwarp();
        if (p.S != nullptr)
          tma_gather4(sA + s * kLinABytes + 4 * lane * 128, &p.x_map, &full[s], 64 * kc, y[0], y[1], y[2], y[3]);
        issued = g + 1;
      }
    }
    if ((!ok || abort_flag) && lane == 0) {
      // let every copy this CTA started land before it exits
      for (int g = issued - ST < 0 ? 0 : issued - ST; g < issued; ++g) mbar_wait_drain(&full[g % ST], (g / ST) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t leader = elect_one_sync();
    constexpr uint32_t idesc = make_idesc_bf16(128, 256, 0, 0);
    bool ok = true;
    for (int i = 0; i < n_local && ok; ++i) {
      const int a = i & 1;
      if (i >= 2 && !warp_wait(&acc_empty[a], ((i >> 1) - 1) & 1, &abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tacc = tbase + 256u * a;
      for (int kc = 0; kc < nk; ++kc) {
        const int g = i * nk + kc, s = g % ST;
        if (!warp_wait(&full[s], (g / ST) & 1, &abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * kLinABytes), b0 = smem_u32(sB + s * kLinBBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ss_if(leader, tacc, make_sdesc(a0 + 32 * kk, 16, 1024, kSwizzle128B),
                     make_sdesc(b0 + 32 * kk, 16, 1024, kSwizzle128B), idesc, (kc | kk) != 0 ? 1u : 0u);
        umma_commit_if(leader, &empty[s]);  // the stage may be refilled once these MMAs have read it
      }
      if (ok) umma_commit_if(leader, &acc_full[a]);
    }
    if (!ok) {
      // wait for every MMA the leader issued before TMEM is released
      umma_commit_if(leader, drain);
      if (leader) mbar_wait_drain(drain, 0);
      __syncwarp();
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3, row = q * 32 + lane, e = (warp - 4) >> 2;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    for (int i = 0; i < n_local; ++i) {
      const int a = i & 1;
      if (!warp_wait(&acc_full[a], (i >> 1) & 1, &abort_flag)) break;
      tc_fence_after();
      int b, r0, n0;
      tile_coords(i, b, r0, n0);
      const int r = r0 + row;
      const bool valid = r < p.R;
      __nv_bfloat16* yrow = p.Y + (static_cast<size_t>(b) * p.R + (valid ? r : 0)) * p.d_out;
      linear_epilogue_tile(p, tbase + lane_addr + 256u * a, e, n0, yrow, valid, [&] { mbar_arrive(&acc_empty[a]); });
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tbase, 512);
}

// The same layer on CTA pairs (clusters of 2, tcgen05 cta_group::2), for the
// plain-rows form (every row of X in order: a compact copy of the rows of S,
// or the dense block). A pair computes a 256 x 256 output tile: the even CTA
// (rank 0) issues M = 256, N = 256, K = 16 MMAs whose A rows 0..127 and B
// rows (output columns) 0..127 come from its own shared memory and rows
// 128..255 from its partner's, at the same offsets; each CTA's TMEM holds its
// 128 output rows x 256 columns. Per 64-wide K chunk each CTA copies 16 KB
// of X and 16 KB of W (against 48 KB per 128 x 256 tile on one SM), so a
// stage is 32 KB and the ring has 6 of them.
//   warp 0     producer in both CTAs: the CTA's X rows and W rows of the
//              chunk, counted on the even CTA's stage barrier
//   warp 1     MMA issuer (even CTA only)
//   warp 2     TMEM allocation (both CTAs, pair form)
//   warps 4..11 epilogue in both CTAs (the CTA's 128 rows, two column halves)
// Barriers: full[s] of the even CTA takes both CTAs' copies (64 KB);
// empty[s] of each CTA is arrived on by the even CTA's MMA commit (the
// stage of both CTAs may be refilled); acc_full[a] the same for the
// accumulator; acc_empty[a] of the even CTA counts the 512 epilogue threads
// of the pair once they have read the accumulator. Every wait is bounded.
constexpr int kLin2Stages = 6;
constexpr int kLin2ABytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kLin2BBytes = 128 * 128;  // 128 W rows x 64 bf16
constexpr int kLin2Smem = 1024 + kLin2Stages * (kLin2ABytes + kLin2BBytes) + 256;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kLinThreads, 1)
    linear_pair_kernel(const __grid_constant__ LinearParams p) {
  constexpr int ST = kLin2Stages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = sm;
  uint8_t* sB = sA + ST * kLin2ABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + ST * kLin2BBytes);  // [ST] both CTAs' stage loaded (rank 0)
  uint64_t* empty = full + ST;                                           // [ST] stage consumed
  uint64_t* acc_full = empty + ST;                                       // [2] accumulator complete
  uint64_t* acc_empty = acc_full + 2;                                    // [2] accumulator read back (rank 0)
  uint64_t* drain = acc_empty + 2;                                       // MMA abort path
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int nk = (p.d_in + 63) / 64;
  const int pair = static_cast<int>(blockIdx.x >> 1), n_pairs = static_cast<int>(gridDim.x >> 1);
  // 256 x 256 tiles of this pair: t = pair + i * n_pairs (column tile fastest)
  const int n_local = p.tiles > pair ? (p.tiles - 1 - pair) / n_pairs + 1 : 0;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 512);  // every epilogue thread of both CTAs
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 2) tmem_alloc_pair(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the partner's barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  auto tile_coords = [&](int i, int& b, int& r0, int& n0) {
    const int t = pair + i * n_pairs;
    const int nt = t % p.n_tiles, mt = t / p.n_tiles;
    b = mt / p.m_tiles;
    r0 = (mt % p.m_tiles) * 256;
    n0 = nt * 256;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      tma_prefetch_desc(&p.xt_map);
      tma_prefetch_desc(&p.w2_map);
    }
    const uint32_t full0 = cluster_addr(full, 0);  // the even CTA's stage barriers
    int issued = 0;
    bool ok = true;
    for (int i = 0; i < n_local && ok; ++i) {
      int b, r0, n0;
      tile_coords(i, b, r0, n0);
      for (int kc = 0; kc < nk; ++kc) {
        const int g = i * nk + kc, s = g % ST;
        if (g >= ST && !warp_wait(&empty[s], ((g / ST) - 1) & 1, &abort_flag)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * (kLin2ABytes + kLin2BBytes));
          const uint32_t bar = full0 + static_cast<uint32_t>(s * sizeof(uint64_t));
          // this CTA's 128 W rows (output columns n0 + 128 rank ..) and 128
          // X rows (r0 + 128 rank ..; rows past the sample's end are other
          // samples' rows or the zero fill past the tensor, not stored)
          tma_load_2d_pair(sB + s * kLin2BBytes, &p.w2_map, bar, 64 * kc, n0 + 128 * static_cast<int>(rank));
          tma_load_2d_pair(sA + s * kLin2ABytes, &p.xt_map, bar, 64 * kc, b * p.N + r0 + 128 * static_cast<int>(rank));
        }
        __syncwarp();
        issued = g + 1;
      }
    }
    if ((!ok || abort_flag) && lane == 0 && rank == 0) {
      // let every copy of the pair land before the CTAs exit
      for (int g = issued - ST < 0 ? 0 : issued - ST; g < issued; ++g) mbar_wait_drain(&full[g % ST], (g / ST) & 1);
    }
  } else if (warp == 1 && rank == 0) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    const uint32_t leader = elect_one_sync();
    constexpr uint32_t idesc = make_idesc_bf16(256, 256, 0, 0);
    const uint32_t empty0 = cluster_addr(empty, 0), empty1 = cluster_addr(empty, 1);
    const uint32_t accf0 = cluster_addr(acc_full, 0), accf1 = cluster_addr(acc_full, 1);
    bool ok = true;
    for (int i = 0; i < n_local && ok; ++i) {
      const int a = i & 1;
      if (i >= 2 && !warp_wait(&acc_empty[a], ((i >> 1) - 1) & 1, &abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tacc = tbase + 256u * a;
      for (int kc = 0; kc < nk; ++kc) {
        const int g = i * nk + kc, s = g % ST;
        if (!warp_wait(&full[s], (g / ST) & 1, &abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * kLin2ABytes), b0 = smem_u32(sB + s * kLin2BBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_pair_ss_if(leader, tacc, make_sdesc(a0 + 32 * kk, 16, 1024, kSwizzle128B),
                          make_sdesc(b0 + 32 * kk, 16, 1024, kSwizzle128B), idesc, (kc | kk) != 0 ? 1u : 0u);
        // both CTAs' stage may be refilled once these MMAs have read it
        const uint32_t so = static_cast<uint32_t>(s * sizeof(uint64_t));
        umma_pair_commit_if(leader, empty0 + so);
        umma_pair_commit_if(leader, empty1 + so);
      }
      if (ok) {
        const uint32_t ao = static_cast<uint32_t>(a * sizeof(uint64_t));
        umma_pair_commit_if(leader, accf0 + ao);
        umma_pair_commit_if(leader, accf1 + ao);
      }
    }
    if (!ok) {
      // wait for every MMA the leader issued before TMEM is released
      umma_pair_commit_if(leader, cluster_addr(drain, 0));
      if (leader) mbar_wait_drain(drain, 0);
      __syncwarp();
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3, row = q * 32 + lane, e = (warp - 4) >> 2;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t acce0 = cluster_addr(acc_empty, 0);
    for (int i = 0; i < n_local; ++i) {
      const int a = i & 1;
      if (!warp_wait(&acc_full[a], (i >> 1) & 1, &abort_flag)) break;
      tc_fence_after();
      int b, r0, n0;
      tile_coords(i, b, r0, n0);
      const int r = r0 + 128 * static_cast<int>(rank) + row;
      const bool valid = r < p.R;
      __nv_bfloat16* yrow = p.Y + (static_cast<size_t>(b) * p.R + (valid ? r : 0)) * p.d_out;
      // the accumulator is released to the even CTA's issuer
      linear_epilogue_tile(p, tbase + lane_addr + 256u * a, e, n0, yrow, valid,
                           [&] { mbar_arrive_cluster(acce0 + static_cast<uint32_t>(a * sizeof(uint64_t))); });
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the partner's MMAs, copies and arrivals are done
  tc_fence_after();
  if (warp == 2) tmem_dealloc_pair(tbase, 512);
}

}  // namespace safe
