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
//   warps 1, 2   MMA issuers (one thread each; tile 0 / tile 1): S_t = Q_t K_j^T
//                into TMEM (SS form), O_t += P_t V_j with P read from TMEM
//                (TS form). With D = 128 warp 1 issues for both tiles.
//   warp 3       assembled-key SRSU only (kAsm): the key / value tiles come
//                from the context cache by TMA, and this warp overwrites in
//                each stage the rows of S with the current rows before the
//                MMA issuers may read it (Eq. (16): K and V of S u C in token
//                order, from current sensitive and cached context rows);
//                otherwise idle (it completes warpgroup 0)
//   warps 4..7   softmax of tile 0, warps 8..11 softmax of tile 1: one
//                thread per query row (one TMEM lane); running max / sum in
//                registers; O rescaled lazily; final O = O_t / l (bf16) and
//                the log-sum-exp.
//
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D),
// O1 [256+D,256+2D), then P (bf16 pairs, 64 columns for 128 keys):
//   D = 64:  one P buffer per tile; each tile only waits for its own P V;
//   D = 96:  one P buffer shared by the two tiles, written in strict
//            alternation P0_j, P1_j, P0_{j+1}, ... (each write waits for the
//            other tile's previous P V, which also orders the O rescale);
//   D = 128: no room: P overwrites S_t and the next S_t follows P_t V.
// With a separate P buffer the softmax releases S_t as soon as it has loaded
// it, so S_t for the next key tile is computed while it exponentiates.
//
// The two tiles' softmax warps of one SM sub-partition (warps 4 + q and
// 8 + q) share its exp unit and take turns on it (named barriers): one
// exponentiates a whole key tile while the other stores P, waits for its next
// S, loads it and takes the row max. The exponentials of a key tile run as
// one pass of 128 independent instructions so that one warp keeps the unit
// busy on its own.
//
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
  // Q and K tiles (K-major operands): chunk c holds columns [64c, 64c +
  // width(c)); 64-wide chunks use the 128B swizzle (128-byte rows), the
  // 32-wide tail of D = 96 the 64B swizzle.
  __host__ __device__ static constexpr int width(int c) { return (D - 64 * c) >= 64 ? 64 : (D - 64 * c); }
  __host__ __device__ static constexpr int row_bytes(int c) { return width(c) * 2; }
  __host__ __device__ static constexpr uint32_t chunk_off(int c) { return static_cast<uint32_t>(c) * 128u * 128u; }
  __host__ __device__ static constexpr uint32_t swizzle(int c) { return width(c) == 64 ? kSwizzle128B : kSwizzle64B; }
  // V tiles (B operand of P V, MN-major) use equal-width chunks so that one
  // MMA with N = D covers the whole head dim: 32-wide with the 64B swizzle
  // for D = 96, 64-wide with the 128B swizzle otherwise; the descriptor's
  // leading byte offset steps from one chunk to the next.
  static constexpr int kVW = (D == 96) ? 32 : 64;
  static constexpr int kVChunks = D / kVW;
  static constexpr uint32_t kVChunkBytes = 128u * kVW * 2u;
  static constexpr uint32_t kVSwizzle = kVW == 32 ? kSwizzle64B : kSwizzle128B;
  // TMEM columns: O_t at kColO + t D; P_t at kColP (+ 64 t with one P
  // buffer per tile) when P has a buffer of its own (kSepP), else in S_t
  static constexpr bool kPerTileP = 256 + 2 * D + 128 <= 512;
  static constexpr bool kSepP = 256 + 2 * D + 64 <= 512;
  static constexpr uint32_t kColO = 256, kColP = 256 + 2 * D;
  __host__ __device__ static constexpr uint32_t col_p(int t) {
    return kSepP ? kColP + (kPerTileP ? 64u * t : 0u) : 128u * t;
  }
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
// descriptor of the 16-key step kk covering all D columns.
template <int D>
__device__ __forceinline__ uint64_t vmajor_desc(uint32_t tile, int kk) {
  using C = TileCfg<D>;
  return make_sdesc(tile + static_cast<uint32_t>(kk * 16 * C::kVW * 2), C::kVChunkBytes, 8 * C::kVW * 2,
                    C::kVSwizzle);
}

struct FlashParams {
  CUtensorMap q_map[2];   // 4-D [B, rows, H, D] map per chunk (dense / compact Q)
  CUtensorMap qg_map[2];  // 2-D [B*N, H*D] gather map per chunk (rows of S)
  CUtensorMap k_map[2];   // 4-D [B, N, H, D]
  CUtensorMap v_map;      // 4-D [B, N, H, D] V map, box kVW wide (chunk chosen by x)
  CUtensorMap o_map[2];   // 4-D [B, n_q, H, D] map of O per chunk (output tile stores)
  const int32_t* S;       // [B, n_q] query rows when gathering, else null
  __nv_bfloat16* O;       // [B, n_q, H, D]
  float* lse;             // [B, H, n_q] or null
  int B, N, H, n_q;
  float scale_log2;       // logit scale * log2(e)
  int gather;
  // assembled-key mode: the current K / V rows of S, [B, n_q, H, D]
  // (cur_compact = 1, row r holds token S[b, r]) or [B, N, H, D]
  const __nv_bfloat16* k_cur;
  const __nv_bfloat16* v_cur;
  int cur_compact;
  // Work units are (b, h, 256-row block), ordered with the row block
  // fastest. The first `full_units` CTAs take one whole unit each; the
  // remaining units are split along the key range into `split` parts, one
  // CTA each, whose partial results flash_merge_kernel combines (balances
  // the last, partial wave of CTAs).
  int n_mblk, full_units, split;
  // part `part` of tail unit `tu` is slot tu * split + part: its rows' O / l
  // in bf16 ([slots * 256, D], written by TMA stores through ws_map, a 4-D
  // [1, slots * 256, 1, D] view) and (running max in log2 units, row sum)
  __nv_bfloat16* ws_ob;
  float2* ws_ml;
  CUtensorMap ws_map[2];
};

constexpr int kFlashThreads = 640;
// Register split after setmaxnreg: warpgroup 0 (producer, MMA issuers)
// keeps kFlashRegsControl, the four softmax warpgroups get
// kFlashRegsSoftmax: 128 * 64 + 512 * 104 = 61440 = 640 * 96, the
// allocation the kernel is launched with (at most 96 per thread). With 64
// (not 40) the issue loops compile without spills.
constexpr uint32_t kFlashRegsControl = 64, kFlashRegsSoftmax = 104;
// Shared by the cross-attention kernel (384 threads, 168 per thread at
// launch): 128 * 104 + 256 * 200 = 384 * 168.
constexpr uint32_t kRegsControl = 104, kRegsSoftmax = 200;

template <int D>
__host__ __device__ constexpr int flash_smem_bytes() {
  using C = TileCfg<D>;
  return 1024 /*align slack*/ + (2 + 2 * C::kStages) * C::kTileBytes + 512 /*barriers + tmem slot*/;
}

// Most key-range parts a split unit is cut into (the planner's limit).
constexpr int kMaxSplit = 16;

// Combines the key-range parts of the split units: one warp per query row,
// lane l owns columns [4l, 4l + 4):
//   M = max_i m_i,  L = sum_i 2^(m_i - M) l_i,  O = sum_i 2^(m_i - M) O_i / L
template <int D>
__global__ void __launch_bounds__(256) flash_merge_kernel(const __grid_constant__ FlashParams p, int tail_units) {
  pdl_wait();  // every part of the attention launch is stored
  const int lane = threadIdx.x & 31;
  const int wid = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (wid >= tail_units * 256) return;
  const int tu = wid / 256, r = wid % 256;
  const int unit = p.full_units + tu;
  const int h = (unit / p.n_mblk) % p.H, b = unit / (p.n_mblk * p.H);
  const int qr = (unit % p.n_mblk) * 256 + r;
  if (qr >= p.n_q) return;
  const size_t slot0 = static_cast<size_t>(tu) * p.split * 256 + r;
  // every part's (m, l) and O slice requested at once (at most kMaxSplit
  // parts), then combined
  const bool active = lane < D / 4;
  float2 ml[kMaxSplit];
  uint2 x[kMaxSplit];  // four bf16 of O_i / l_i
#pragma unroll
  for (int i = 0; i < kMaxSplit; ++i) {
    ml[i] = make_float2(-INFINITY, 0.f);
    x[i] = make_uint2(0u, 0u);
    if (i < p.split) {
      const size_t slot = slot0 + static_cast<size_t>(i) * 256;
      ml[i] = __ldcg(&p.ws_ml[slot]);
      if (active) x[i] = __ldcg(reinterpret_cast<const uint2*>(p.ws_ob + slot * D) + lane);
    }
  }
  float M = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMaxSplit; ++i) M = fmaxf(M, ml[i].x);
  // O = sum_i 2^(m_i - M) l_i (O_i / l_i) / L,  L = sum_i 2^(m_i - M) l_i
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < kMaxSplit; ++i) {
    if (i < p.split) {
      const float w = ex2_approx(ml[i].x - M) * ml[i].y;
      L += w;
      acc.x = fmaf(w, __uint_as_float(x[i].x << 16), acc.x);
      acc.y = fmaf(w, __uint_as_float(x[i].x & 0xFFFF0000u), acc.y);
      acc.z = fmaf(w, __uint_as_float(x[i].y << 16), acc.z);
      acc.w = fmaf(w, __uint_as_float(x[i].y & 0xFFFF0000u), acc.w);
    }
  }
  const float inv_l = 1.f / L;
  if (active) {
    __nv_bfloat16* orow = p.O + ((static_cast<size_t>(b) * p.n_q + qr) * p.H + h) * D;
    reinterpret_cast<uint2*>(orow)[lane] =
        make_uint2(pack_bf16x2(acc.x * inv_l, acc.y * inv_l), pack_bf16x2(acc.z * inv_l, acc.w * inv_l));
  }
  if (lane == 0 && p.lse != nullptr)
    p.lse[(static_cast<size_t>(b) * p.H + h) * p.n_q + qr] = (M + __log2f(L)) * 0.69314718055994531f;
}

__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) return false;
  }
  return true;
}

// Warp-uniform bounded wait (every lane polls; all agree on the outcome
// before a warp-collective tcgen05 instruction follows).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
}

// Byte offset, inside a K stage buffer (K-major chunks, see TileCfg), of the
// 16-byte unit u (head-dim columns [8u, 8u + 8)) of key row r, with the
// chunk's swizzle applied as the TMA copy of the tile applies it: the unit
// index XOR (r mod 8) for 128-byte rows, XOR ((r / 2) mod 4) for 64-byte rows.
template <int D>
__device__ __forceinline__ uint32_t k_unit_off(int r, int u) {
  using C = TileCfg<D>;
  const int c = u >> 3, uc = u & 7;
  const int rb = C::row_bytes(c);
  const int xr = rb == 128 ? (r & 7) : ((r >> 1) & 3);
  return C::chunk_off(c) + static_cast<uint32_t>(r * rb + ((uc ^ xr) << 4));
}

// The same for a V stage buffer (equal-width MN-major chunks of kVW columns).
template <int D>
__device__ __forceinline__ uint32_t v_unit_off(int r, int u) {
  using C = TileCfg<D>;
  constexpr int U = C::kVW / 8;  // units per chunk row
  const int c = u / U, uc = u % U;
  const int xr = U == 8 ? (r & 7) : ((r >> 1) & 3);
  return static_cast<uint32_t>(c) * C::kVChunkBytes + static_cast<uint32_t>(r * C::kVW * 2 + ((uc ^ xr) << 4));
}

// Assembled-key mode, run by one warp: for each key tile of the CTA, wait for
// the cache copy of K_j and V_j, overwrite the rows that belong to S with the
// current rows, and release the stage (k_ready, v_ready). S is ascending, so
// the rows of S inside tile j are one run of S that starts where the previous
// tile's run ended (the first run by binary search); each lane copies one row
// of a 32-row round of the run. A row is checked to lie inside the tile
// before it is copied (a row out of order is skipped and flagged).
// Stage j - 1 is released after stage j's copies are issued when K_j / V_j
// have already landed (its copy latency then overlaps that work), else
// before waiting for them: a release never waits for a TMA copy, so the
// stages cannot wait on each other in a cycle, and the prefetch depth of the
// ring is kept.
template <int D>
__device__ void assemble_current_rows(const FlashParams& p, uint8_t* sK, uint8_t* sV, uint64_t* k_full,
                                      uint64_t* v_full, uint64_t* k_ready, uint64_t* v_ready, int b, int h, int kv0,
                                      int n_kv, volatile int* abort) {
  using C = TileCfg<D>;
  constexpr int ST = C::kStages, TB = C::kTileBytes, UPR = D / 8;
  const int lane = threadIdx.x & 31;
  const int32_t* Sb = p.S + static_cast<size_t>(b) * p.n_q;
  const size_t pitch = static_cast<size_t>(p.H) * D;  // elements from one token row to the next
  const size_t base = static_cast<size_t>(b) * (p.cur_compact ? p.n_q : p.N) * pitch + static_cast<size_t>(h) * D;
  const __nv_bfloat16* kb = p.k_cur + base;
  const __nv_bfloat16* vb = p.v_cur + base;
  // the copies are generic-proxy writes: each lane waits for its own, fences
  // them towards the tensor cores' async proxy and then arrives
  auto release = [&](int stage) {
    fence_proxy_async_smem();
    mbar_arrive(&k_ready[stage]);
    mbar_arrive(&v_ready[stage]);
  };
  // first entry of S at or after this CTA's first key
  int lo = 0, hi = p.n_q;
  const int first = kv0 * 128;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(Sb + mid) < first)
      lo = mid + 1;
    else
      hi = mid;
  }
  int cur = lo;
  bool bad = false, ok = true;
  // first round of each tile's run: entry cur + lane of S, loaded ahead
  int i = cur + lane;
  int key = i < p.n_q ? __ldg(Sb + i) : INT_MAX;
  for (int j = 0; j < n_kv; ++j) {
    const int s = j % ST;
    const uint32_t par = (j / ST) & 1;
    const int j0 = (kv0 + j) * 128;
    const int lim = j0 + 128 < p.N ? j0 + 128 : p.N;
    bool prev_open = j > 0;  // stage j - 1 not yet released
    if (prev_open) {
      const int landed = lane == 0 ? static_cast<int>(mbar_test(&k_full[s], par) && mbar_test(&v_full[s], par)) : 0;
      if (!__shfl_sync(0xffffffffu, landed, 0)) {
        cp_async_wait<0>();
        release((j - 1) % ST);
        prev_open = false;
      }
    }
    if (!warp_wait(&k_full[s], par, abort) || !warp_wait(&v_full[s], par, abort)) {
      ok = false;
      break;
    }
    const uint32_t k_dst = smem_u32(sK + s * TB), v_dst = smem_u32(sV + s * TB);
    for (;;) {
      const unsigned in = __ballot_sync(0xffffffffu, key < lim);
      const int run = in == 0xffffffffu ? 32 : __ffs(~in) - 1;  // leading lanes inside the tile
      if (lane < run) {
        const int r = key - j0;  // key < lim holds for these lanes
        if (r < 0) {
          bad = true;
        } else {
          const size_t row = p.cur_compact ? static_cast<size_t>(i) : static_cast<size_t>(key);
          const __nv_bfloat16* ks = kb + row * pitch;
          const __nv_bfloat16* vs = vb + row * pitch;
#pragma unroll
          for (int u = 0; u < UPR; ++u) cp_async16(k_dst + k_unit_off<D>(r, u), ks + 8 * u);
#pragma unroll
          for (int u = 0; u < UPR; ++u) cp_async16(v_dst + v_unit_off<D>(r, u), vs + 8 * u);
        }
      }
      cur += run;
      i = cur + lane;
      key = i < p.n_q ? __ldg(Sb + i) : INT_MAX;  // next round, or the next tile's first
      if (run < 32) break;
    }
    cp_async_commit();
    if (prev_open) {
      cp_async_wait<1>();  // every group but this stage's
      release((j - 1) % ST);
    }
  }
  cp_async_wait<0>();
  if (ok && n_kv > 0) release((n_kv - 1) % ST);
  if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(1 << 5);
}

template <int D, bool kAsm>
__global__ void __launch_bounds__(kFlashThreads, 1) flash_fwd_kernel(const __grid_constant__ FlashParams p) {
  using C = TileCfg<D>;
  constexpr int ST = C::kStages;
  constexpr int TB = C::kTileBytes;
  constexpr bool kSepP = C::kSepP;
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
  uint64_t* s_full = kv_empty + ST;  // [2] S_t computed
  uint64_t* s_free = s_full + 2;     // [2] S_t loaded by the softmax (separate-P mode)
  uint64_t* p_full = s_free + 2;     // [2] P_t written
  uint64_t* pv_done = p_full + 2;    // [2] P_t V complete (separate-P mode)
  uint64_t* o_full = pv_done + 2;    // [2] last P_t V complete
  uint64_t* drain = o_full + 2;      // [2] per MMA issuer, abort path only
  uint64_t* k_ready = drain + 2;     // [ST] assembled mode: rows of S written into K_j (32 arrivals)
  uint64_t* v_ready = k_ready + ST;  // [ST] ... and into V_j
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(v_ready + ST);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_kv_all = (p.N + 127) / 128;
  int unit = blockIdx.x, tail_u = 0, part = 0, kv0 = 0, kv1 = n_kv_all;
  if (unit >= p.full_units) {
    const int k = unit - p.full_units;
    tail_u = k / p.split;
    part = k % p.split;
    unit = p.full_units + tail_u;
    kv0 = part * n_kv_all / p.split;
    kv1 = (part + 1) * n_kv_all / p.split;
  }
  const bool partial = p.split > 1 && blockIdx.x >= p.full_units;
  const int h = (unit / p.n_mblk) % p.H, b = unit / (p.n_mblk * p.H);
  const int q_base = (unit % p.n_mblk) * 256;
  const int n_kv = kv1 - kv0;  // key tiles of this CTA: [kv0, kv1)

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], kSepP ? 2 : 1);  // one commit per MMA issuer
      mbar_init(&k_ready[s], 32);  // every lane of the assembling warp
      mbar_init(&v_ready[s], 32);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&s_free[t], 256);  // both column halves of the tile's 128 rows
      mbar_init(&p_full[t], 256);
      mbar_init(&pv_done[t], 1);
      mbar_init(&o_full[t], 1);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  // launched as a programmatic dependent: the set-up above overlapped the
  // previous kernel; its outputs (the inputs here) are read only from now on
  pdl_launch_dependents();
  pdl_wait();

  if (warp < 4) {
    regs_dealloc<kFlashRegsControl>();
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0) {
        for (int c = 0; c < C::kChunks; ++c) tma_prefetch_desc(&p.k_map[c]);
        tma_prefetch_desc(&p.v_map);
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
            tma_load_4d(sK + s * TB + C::chunk_off(c), &p.k_map[c], &k_full[s], 64 * c, h, (kv0 + j) * 128, b);
          mbar_arrive_expect_tx(&v_full[s], TB);
          for (int c = 0; c < C::kVChunks; ++c)
            tma_load_4d(sV + s * TB + c * C::kVChunkBytes, &p.v_map, &v_full[s], C::kVW * c, h, (kv0 + j) * 128, b);
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
    } else if (warp == 1 || (kSepP && warp == 2)) {
      // ---------------------------------------------------------- MMA issuers
      // separate-P mode: warp 1 issues tile 0's MMAs and warp 2 tile 1's
      // (tcgen05.commit tracks the issuing thread's MMAs, so each issuer
      // signals its own tile); aliased mode: warp 1 issues both tiles. Each
      // issuing warp runs its loop with all lanes and one elected lane issues.
      {
        // the whole warp runs the issue loop; the elected lane issues
        const uint32_t leader = elect_one_sync();
        const int mt = warp - 1;  // tile of this issuer (separate-P mode)
        constexpr uint32_t idS = make_idesc_bf16(128, 128, 0, 0);
        constexpr uint32_t idPV = make_idesc_bf16(128, D, 0, 1);
        constexpr int KS = D / 16;
        // TMEM column of S_t, O_t and P_t (t = 0, 1)
        auto tS = [&](int t) -> uint32_t { return tbase + 128u * t; };
        auto tO = [&](int t) -> uint32_t { return tbase + C::kColO + static_cast<uint32_t>(D) * t; };
        auto tP = [&](int t) -> uint32_t { return tbase + C::col_p(t); };
        // stage barriers the MMAs wait on: the TMA copy, or, with assembled
        // keys, the rows of S written over it
        uint64_t* k_in = kAsm ? k_ready : k_full;
        uint64_t* v_in = kAsm ? v_ready : v_full;
        // Descriptors of stage 0 / k-step 0; a k-step or a stage only moves
        // the start address (low 14 bits, in 16-byte units), so each MMA
        // adds a constant to the low word.
        const uint64_t dQ0 = kmajor_desc<D>(smem_u32(sQ), 0), dQ1 = kmajor_desc<D>(smem_u32(sQ + TB), 0);
        const uint64_t dK = kmajor_desc<D>(smem_u32(sK), 0);
        const uint64_t dV = vmajor_desc<D>(smem_u32(sV), 0);
        auto koff = [](int kk) -> uint32_t { return (C::chunk_off(kk >> 2) + (kk & 3) * 32) >> 4; };
        // the two K-major chunks of D = 96 differ in swizzle: take the high
        // word (layout, strides) per chunk, the start address from the base
        auto kdesc = [&](uint64_t base, int kk, uint32_t so) -> uint64_t {
          const uint64_t hi = kmajor_desc<D>(0, kk) & 0xFFFFFFFF00000000ull;
          return hi | static_cast<uint32_t>(static_cast<uint32_t>(base) + koff(kk) + so);
        };
        auto issue_S = [&](int t, int s) {
          const uint32_t so = static_cast<uint32_t>((s * TB) >> 4);
          const uint64_t dq = t == 0 ? dQ0 : dQ1;
#pragma unroll
          for (int kk = 0; kk < KS; ++kk)
            umma_ss_if(leader, tS(t), kdesc(dq, kk, 0), kdesc(dK, kk, so), idS, kk > 0 ? 1u : 0u);
        };
        // O_t (+)= P_t V: 8 steps of 16 keys, one N = D instruction each
        auto issue_PV = [&](int t, int s, int j) {
          const uint32_t so = static_cast<uint32_t>((s * TB) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t v = static_cast<uint32_t>(dV) + so + ((kk * 16 * C::kVW * 2) >> 4);
            umma_ts_if(leader, tO(t), tP(t) + kk * 8, (dV & 0xFFFFFFFF00000000ull) | v, idPV,
                       (j > 0 || kk > 0) ? 1u : 0u);
          }
        };
        bool ok = warp_wait(q_full, 0, &abort_flag) && warp_wait(&k_in[0], 0, &abort_flag);
        if (ok) {
          tc_fence_after();
          if constexpr (kSepP) {
            // per tile: the next S as soon as the softmax has loaded the
            // current one, then P V once P is written
            issue_S(mt, 0);
            umma_commit_if(leader, &s_full[mt]);
            for (int j = 0; j < n_kv && ok; ++j) {
              const int s = j % ST;
              if (j + 1 < n_kv) {
                const int s1 = (j + 1) % ST;
                ok = warp_wait(&k_in[s1], ((j + 1) / ST) & 1, &abort_flag) &&
                     warp_wait(&s_free[mt], j & 1, &abort_flag);
                if (!ok) break;
                tc_fence_after();
                issue_S(mt, s1);
                umma_commit_if(leader, &s_full[mt]);
              }
              ok = warp_wait(&v_in[s], (j / ST) & 1, &abort_flag) && warp_wait(&p_full[mt], j & 1, &abort_flag);
              if (!ok) break;
              tc_fence_after();
              issue_PV(mt, s, j);
              umma_commit_if(leader, &pv_done[mt]);
              umma_commit_if(leader, &kv_empty[s]);  // this tile no longer reads K_j, V_j
              if (j + 1 == n_kv) umma_commit_if(leader, &o_full[mt]);
            }
          } else {
          issue_S(0, 0);
          umma_commit_if(leader, &s_full[0]);
          issue_S(1, 0);
          umma_commit_if(leader, &s_full[1]);
          for (int j = 0; j < n_kv && ok; ++j) {
            const int s = j % ST;
            {
              // P overwrites S_t: the next S_t follows P_t V
              ok = warp_wait(&v_in[s], (j / ST) & 1, &abort_flag);
              for (int t = 0; t < 2 && ok; ++t) {
                ok = warp_wait(&p_full[t], j & 1, &abort_flag);
                if (!ok) break;
                tc_fence_after();
                issue_PV(t, s, j);
                if (j + 1 < n_kv) {
                  const int s1 = (j + 1) % ST;
                  if (t == 0) {
                    ok = warp_wait(&k_in[s1], ((j + 1) / ST) & 1, &abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                  }
                  issue_S(t, s1);
                  umma_commit_if(leader, &s_full[t]);
                } else {
                  umma_commit_if(leader, &o_full[t]);
                }
              }
            }
            if (ok) umma_commit_if(leader, &kv_empty[s]);
          }
          }
        }
        if (!ok) {
          // wait for every MMA the leader issued before TMEM is released
          umma_commit_if(leader, &drain[warp - 1]);
          mbar_wait_drain(&drain[warp - 1], 0);
        }
      }
    } else if (kAsm && warp == 3) {
      // ---------------------------------------------------------- rows of S
      assemble_current_rows<D>(p, sK, sV, k_full, v_full, k_ready, v_ready, b, h, kv0, n_kv, &abort_flag);
    }
  } else {
    regs_alloc<kFlashRegsSoftmax>();
    // ------------------------------------------------------------ softmax
    // Warp 4 + 4 g + q, g = 2 t + hf: query rows 32 q .. 32 q + 31 of tile
    // t (TMEM lanes of sub-partition q), keys 64 hf .. 64 hf + 63 of each key
    // tile (the column half hf of S and of P) and columns hf D/2 .. of O.
    const int g = (warp - 4) >> 2, t = g >> 1, hf = g & 1;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tbase + lane_addr + t * 128 + 64 * hf;
    constexpr int DH = D / 2;  // O columns of one half
    const uint32_t tO = tbase + lane_addr + C::kColO + t * D + DH * hf;
    const uint32_t tP = tbase + lane_addr + C::col_p(t) + 32 * hf;
    const int q_row = q_base + t * 128 + row;
    const float sl2 = p.scale_log2;
    // valid keys of this half in this CTA's last key tile (fewer than 64
    // only in the global last tile)
    const int tail = (kv1 == n_kv_all ? p.N - (n_kv_all - 1) * 128 : 128) - 64 * hf;
    float m_use = -INFINITY, l = 0.f;
    bool ok = true;
    // The four softmax warps of one SM sub-partition share its exp unit: the
    // two column halves of tile 0 exponentiate together, then the two of
    // tile 1, and so on, each pair loading S, taking its half-row max and
    // storing P while the other pair exponentiates. Named barrier 1 + 2q + t
    // is "tile t may exponentiate" (128 threads: the pair that waits and the
    // pair that hands over); it also publishes the half-row maxima, which
    // each half writes to shared memory before it waits. Every warp takes
    // every barrier step on every path (an abort only skips the work).
    const uint32_t bar_mine = 1 + 2 * quarter + t, bar_other = 1 + 2 * quarter + (1 - t);
    __shared__ float half_max[2][2][2][128];  // [step parity][tile][half][row]
    // store this half of P_t of key tile j (32 bf16 pairs in pk) and rescale
    // this half of O_t first when the running max grew
    auto store_p = [&](int j, const uint32_t* pk, bool need, float alpha) {
      if constexpr (kSepP) {
        // the P buffer is free and O_t idle: one buffer per tile: this
        // tile's previous P V is complete; shared buffer: the other tile's
        // previous P V (P0_j after P1_{j-1} V, P1_j after P0_j V; the
        // other tile's write waited for this tile's previous P V)
        bool w = true;
        if (C::kPerTileP || t == 0) {
          if (j > 0) w = warp_wait(&pv_done[C::kPerTileP ? t : 1], (j - 1) & 1, &abort_flag);
        } else {
          w = warp_wait(&pv_done[0], j & 1, &abort_flag);
        }
        if (!w) {
          ok = false;
          return;
        }
        tc_fence_after();
      }
      // (aliased mode: O_t is idle because P_t V of the previous step
      // completed before S_t of this step was committed)
      if (__any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int c = 0; c < DH / 16; ++c) {
          uint32_t o[16];
          tmem_ld16(tO + 16 * c, o);
          tmem_ld_wait16(o);
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st16(tO + 16 * c, o);
        }
      }
      tmem_st16(tP, pk);
      tmem_st16(tP + 16, pk + 16);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    };
    if (t == 1) named_bar_arrive(bar_other, 128);  // tile 0 goes first
    for (int j = 0; j < n_kv; ++j) {
      // After an abort the arithmetic still runs (on whatever TMEM holds)
      // but no wait, arrival or store is made; the barrier steps stay.
      if (ok) ok = warp_wait(&s_full[t], j & 1, &abort_flag);
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(tS + 0, sr);
      tmem_ld32(tS + 32, sr + 32);
      tmem_ld_wait32(sr);
      tmem_ld_wait32(sr + 32);
      if (kSepP && ok) {
        // this half of S_t is in registers: the MMA issuer may overwrite it
        tc_fence_before();
        mbar_arrive(&s_free[t]);
      }
      if (j == n_kv - 1 && tail < 64) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= tail) sr[c] = __float_as_uint(-INFINITY);
      }
      float mx0 = fmax3(__uint_as_float(sr[0]), __uint_as_float(sr[1]), __uint_as_float(sr[2]));
      float mx1 = fmax3(__uint_as_float(sr[3]), __uint_as_float(sr[4]), __uint_as_float(sr[5]));
      float mx2 = fmax3(__uint_as_float(sr[6]), __uint_as_float(sr[7]), __uint_as_float(sr[8]));
      float mx3 = fmax3(__uint_as_float(sr[9]), __uint_as_float(sr[10]), __uint_as_float(sr[11]));
#pragma unroll
      for (int c = 12; c < 60; c += 8) {
        mx0 = fmax3(mx0, __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
        mx1 = fmax3(mx1, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
        mx2 = fmax3(mx2, __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
        mx3 = fmax3(mx3, __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
      }
      mx0 = fmax3(mx0, __uint_as_float(sr[60]), __uint_as_float(sr[61]));
      mx1 = fmax3(mx1, __uint_as_float(sr[62]), __uint_as_float(sr[63]));
      const float mx = fmax3(mx0, mx1, fmaxf(mx2, mx3));
      half_max[j & 1][t][hf][row] = mx;
      // ---- this tile's turn on the exp unit (and the other half's maximum)
      named_bar_sync(bar_mine, 128);
      const float m_cand = fmaxf(mx, half_max[j & 1][t][hf ^ 1][row]) * sl2;
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
      // probabilities: x = s scale log2(e) - m, then 2^x as one pass of 64
      // independent exponentials, then the row sum and the bf16 pairs
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      const uint64_t negm2 = f2_pack(-m_use, -m_use);
      float x[64];
#pragma unroll
      for (int i = 0; i < 32; ++i)
        f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), sl2x2, negm2),
                  x[2 * i], x[2 * i + 1]);
#pragma unroll
      for (int c = 0; c < 64; ++c) x[c] = ex2_approx(x[c]);
      uint32_t pk[32];
      uint64_t acc0 = 0, acc1 = 0;  // packed row sums (bit pattern 0 = +0.0f)
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint64_t e2 = f2_pack(x[2 * i], x[2 * i + 1]);
        if (i & 1) acc1 = f2_add(acc1, e2); else acc0 = f2_add(acc0, e2);
        pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
      }
      // ---- hand the exp unit to the other tile
      if (t == 0 || j + 1 < n_kv) named_bar_arrive(bar_other, 128);
      if (ok) store_p(j, pk, need, alpha);
      float s0, s1, s2, s3;
      f2_unpack(acc0, s0, s1);
      f2_unpack(acc1, s2, s3);
      l = l * alpha + ((s0 + s1) + (s2 + s3));
    }
    // the row sum is the sum of the two halves' sums (same running max)
    __shared__ float half_sum[2][2][128];
    half_sum[t][hf][row] = l;
    named_bar_sync(9, 512);
    l = half_sum[t][0][row] + half_sum[t][1][row];
    const bool have_o = ok && warp_wait(&o_full[t], 0, &abort_flag);
    if (have_o) tc_fence_after();
    const bool valid = q_row < p.n_q;
    {
      // O / l in bf16 into this tile's query buffer (free: every S product
      // of the tile completed before its last P V), laid out as the query
      // tile was, then one TMA store per head-dim chunk: into O (rows past
      // n_q are clipped by the store), or, for one part of a split unit, into
      // its workspace slot with the rows' running max and sum beside it
      // (flash_merge_kernel combines the parts)
      uint8_t* stage = sQ + t * TB;
      const int slot = partial ? tail_u * p.split + part : 0;
      if (have_o) {
        const float inv_l = 1.f / l;
#pragma unroll
        for (int c = 0; c < DH / 16; ++c) {
          uint32_t o[16];
          tmem_ld16(tO + 16 * c, o);
          tmem_ld_wait16(o);
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const int u = (DH * hf + 16 * c) / 8 + v;  // 16-byte unit of the row
            const int cq = u >> 3, uc = u & 7;
            const int rb = C::row_bytes(cq);
            const int xr = rb == 128 ? (row & 7) : ((row >> 1) & 3);
            *reinterpret_cast<uint4*>(stage + C::chunk_off(cq) + row * rb + ((uc ^ xr) << 4)) =
                make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
        if (partial) {
          if (hf == 0) p.ws_ml[static_cast<size_t>(slot) * 256 + t * 128 + row] = make_float2(m_use, l);
        } else if (valid && hf == 0 && p.lse != nullptr) {
          p.lse[(static_cast<size_t>(b) * p.H + h) * p.n_q + q_row] = (m_use + __log2f(l)) * 0.69314718055994531f;
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(10 + t, 256);  // the tile's eight softmax warps
      if (quarter == 0 && hf == 0 && lane == 0 && !abort_flag && q_base + t * 128 < p.n_q) {
        for (int c = 0; c < C::kChunks; ++c) {
          if (partial)
            tma_store_4d(&p.ws_map[c], stage + C::chunk_off(c), 64 * c, 0, slot * 256 + t * 128, 0);
          else
            tma_store_4d(&p.o_map[c], stage + C::chunk_off(c), 64 * c, h, q_base + t * 128, b);
        }
        bulk_commit_group();
        bulk_wait_read_all();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, 512);
}

}  // namespace safe
