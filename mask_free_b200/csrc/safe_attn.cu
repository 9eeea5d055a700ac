// safe_attn.cu - host side of the C ABI declared in include/safe_attn.h.
//
// One translation unit: it includes every kernel of the library, validates
// arguments on the host, encodes the TMA tensor maps and launches on the
// caller's stream. The library allocates no device memory.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "safe_attn.h"
#include "sm100.cuh"
#include "flash_attn.cuh"
#include "cross_attn.cuh"
#include "aux_kernels.cuh"
#include "guidance.cuh"
#include "linear.cuh"

using namespace safe;

namespace {

constexpr int kAbiVersion = 7;
constexpr float kLog2e = 1.4426950408889634f;

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_d(int d) { return d == 64 || d == 96 || d == 128; }

// The attention kernels take each row's maximum of the unscaled logits and
// scale it afterwards, which is the row's largest scaled logit only for a
// positive scale; padding keys are masked with -inf before scaling.
bool scale_ok(float scale) { return std::isfinite(scale) && scale > 0.f; }

safe_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? SAFE_OK : SAFE_ERR_CUDA;
}

// ---------------------------------------------------------------- TMA maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

int chunk_width(int d, int c) { return (d - 64 * c) >= 64 ? 64 : (d - 64 * c); }

CUtensorMapSwizzle chunk_swizzle(int d, int c) {
  return chunk_width(d, c) == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
}

// [B, rows, H, d] bf16 tensor viewed as 4-D (d, H, rows, B); box = one
// chunk of the head dim x 1 head x 128 rows x 1 sample. Rows past `rows`
// read as zero.
bool encode_rows_map(CUtensorMap* map, const void* base, int B, int rows, int H, int d, int c) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2,
                           static_cast<cuuint64_t>(rows) * H * d * 2};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(chunk_width(d, c)), 1, 128, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, chunk_swizzle(d, c), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Same 4-D view with the equal-width V chunks of the flash kernel (32 wide
// with the 64B swizzle for d = 96, else 64 wide with the 128B swizzle).
bool encode_v_map(CUtensorMap* map, const void* base, int B, int rows, int H, int d) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const int w = d == 96 ? 32 : 64;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2,
                           static_cast<cuuint64_t>(rows) * H * d * 2};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(w), 1, 128, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, w == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [B*N, H*d] 2-D view for tile::gather4 (box one row high).
// 2-D bf16 matrix [outer, inner] (row pitch = inner), 128B swizzle; box
// box_inner x box_outer (the row-wise layers' X, box 64 x 1 for gather4, and
// W^T, box 64 x 256).
bool encode_matrix_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                       uint32_t box_outer) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_gather_map(CUtensorMap* map, const void* base, int B, int N, int H, int d, int c) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(H) * d, static_cast<cuuint64_t>(B) * N};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(H) * d * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(chunk_width(d, c)), 1};
  cuuint32_t es[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, chunk_swizzle(d, c), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int nchunks(int d) { return (d + 63) / 64; }

// ---------------------------------------------------------------- launches
int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return sms;
  static int cached[64] = {};
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cached[dev] = sms;
  return sms;
}

// How the (b, h, 256-row block) work units of one flash launch are spread
// over the SMs: `full` whole units first, then the remaining units split
// into `split` key ranges each (see FlashParams).
struct FlashPlan {
  int units, full, split, tail;
  size_t ws_o, ws_ml, ws_bytes;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

FlashPlan plan_flash(int B, int H, int n_q, int N, int d, int sms) {
  FlashPlan pl{};
  const int n_mblk = (n_q + 255) / 256;
  const int n_kv = (N + 127) / 128;
  pl.units = n_mblk * H * B;
  pl.full = pl.units;
  pl.split = 1;
  pl.tail = 0;
  // Cost model in key-tile steps (calibrated on B200): a whole unit costs
  // n_kv + 2, a part n_kv / s + 8 (set-up, pipeline fill and drain, partial
  // store, and the spread of finish times across SMs), the merge launch
  // about 3. Only the last waves are split; each part keeps at least 4 key
  // tiles.
  const double whole = n_kv + 2.0;
  double best = static_cast<double>((pl.units + sms - 1) / sms) * whole;
  const int max_split = n_kv / 4 < kMaxSplit ? n_kv / 4 : kMaxSplit;  // the merge kernel takes at most kMaxSplit parts
  for (int fw = pl.units / sms; fw >= 0 && fw >= pl.units / sms - 1; --fw) {
    const int f = fw * sms, r = pl.units - f;
    if (r <= 0) continue;
    for (int sp = 2; sp <= max_split; ++sp) {
      const double rounds = static_cast<double>((static_cast<long long>(r) * sp + sms - 1) / sms);
      const double cost = fw * whole + rounds * (static_cast<double>(n_kv) / sp + 8.0) + 3.0;
      if (cost < 0.99 * best) {
        best = cost;
        pl.full = f;
        pl.split = sp;
        pl.tail = r;
      }
    }
  }
  if (pl.split > 1) {
    const size_t slots = static_cast<size_t>(pl.tail) * pl.split * 256;
    pl.ws_o = 0;  // bf16 O / l of the parts
    pl.ws_ml = align256(slots * d * 2);
    pl.ws_bytes = pl.ws_ml + align256(slots * sizeof(float2));
  }
  return pl;
}

template <int D, bool kAsm>
safe_status launch_flash(FlashParams& p, void* ws, size_t ws_bytes, cudaStream_t s) {
  constexpr int smem = flash_smem_bytes<D>();
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(flash_fwd_kernel<D, kAsm>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (attr_err != cudaSuccess) return SAFE_ERR_CUDA;
  FlashPlan pl = plan_flash(p.B, p.H, p.n_q, p.N, D, device_sms());
  if (pl.split > kMaxSplit) return SAFE_ERR_UNSUPPORTED;  // the merge takes at most kMaxSplit parts
  if (pl.split > 1 && (!aligned16(ws) || ws_bytes < pl.ws_bytes)) {
    pl.full = pl.units;  // no workspace: whole units only
    pl.split = 1;
    pl.tail = 0;
  }
  p.n_mblk = (p.n_q + 255) / 256;
  p.full_units = pl.full;
  p.split = pl.split;
  p.ws_ob = nullptr;
  p.ws_ml = nullptr;
  if (pl.split > 1) {
    uint8_t* w = static_cast<uint8_t*>(ws);
    p.ws_ob = reinterpret_cast<__nv_bfloat16*>(w + pl.ws_o);
    p.ws_ml = reinterpret_cast<float2*>(w + pl.ws_ml);
    for (int c = 0; c < nchunks(D); ++c)
      if (!encode_rows_map(&p.ws_map[c], p.ws_ob, 1, pl.tail * pl.split * 256, 1, D, c)) return SAFE_ERR_CUDA;
  }
  const unsigned grid = static_cast<unsigned>(pl.full + pl.tail * pl.split);
  // both launches are programmatic dependents of what precedes them in the
  // stream: their set-up overlaps its tail, and each waits (griddepcontrol)
  // for it before reading anything
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kFlashThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, flash_fwd_kernel<D, kAsm>, p) != cudaSuccess) return SAFE_ERR_CUDA;
  if (pl.split > 1) {
    cfg.gridDim = dim3((pl.tail * 256 + 7) / 8);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    if (cudaLaunchKernelEx(&cfg, flash_merge_kernel<D>, p, pl.tail) != cudaSuccess) return SAFE_ERR_CUDA;
  }
  return launch_status();
}

// assembled: SRSU with the keys of S taken from p.k_cur / p.v_cur
safe_status dispatch_flash(int d, FlashParams& p, void* ws, size_t ws_bytes, cudaStream_t s, bool assembled = false) {
  switch (d) {
    case 64: return assembled ? launch_flash<64, true>(p, ws, ws_bytes, s) : launch_flash<64, false>(p, ws, ws_bytes, s);
    case 96: return assembled ? launch_flash<96, true>(p, ws, ws_bytes, s) : launch_flash<96, false>(p, ws, ws_bytes, s);
    case 128:
      return assembled ? launch_flash<128, true>(p, ws, ws_bytes, s) : launch_flash<128, false>(p, ws, ws_bytes, s);
    default: return SAFE_ERR_UNSUPPORTED;
  }
}

template <int D, bool kSep, bool kO>
cudaError_t cross_smem_attr() {
  return cudaFuncSetAttribute(cross_attn_kernel<D, kSep, kO>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kCrossMaxSmem);
}

template <int D>
safe_status launch_cross(CrossParams& p, cudaStream_t s) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cross_smem_attr<D, false, true>();
    if (attr_err == cudaSuccess) attr_err = cross_smem_attr<D, false, false>();
    if constexpr (D <= 96) {
      if (attr_err == cudaSuccess) attr_err = cross_smem_attr<D, true, true>();
      if (attr_err == cudaSuccess) attr_err = cross_smem_attr<D, true, false>();
    }
  });
  if (attr_err != cudaSuccess) return SAFE_ERR_CUDA;
  // one CTA per SM (each holds all of TMEM), a few per (b, h), each streaming
  // a contiguous range of query tiles
  const int n_tiles = (p.nq + 127) / 128;
  int per_bh = device_sms() / (p.B * p.H);
  per_bh = per_bh < 1 ? 1 : (per_bh > n_tiles ? n_tiles : per_bh);
  p.qs = cross_slots<D>(p.M);
  dim3 grid(per_bh, p.H, p.B);
  const int smem = cross_smem_bytes<D>(p.M);
  const bool o = p.O != nullptr;  // else PCSP partials only
  bool sep = false;
  if constexpr (D <= 96) sep = cross_sep_p<D>(p.M);
  if constexpr (D <= 96) {
    if (sep) {
      if (o)
        cross_attn_kernel<D, true, true><<<grid, kCrossThreads, smem, s>>>(p);
      else
        cross_attn_kernel<D, true, false><<<grid, kCrossThreads, smem, s>>>(p);
    }
  }
  if (!sep) {
    if (o)
      cross_attn_kernel<D, false, true><<<grid, kCrossThreads, smem, s>>>(p);
    else
      cross_attn_kernel<D, false, false><<<grid, kCrossThreads, smem, s>>>(p);
  }
  return launch_status();
}

safe_status dispatch_cross(int d, CrossParams& p, cudaStream_t s) {
  switch (d) {
    case 64: return launch_cross<64>(p, s);
    case 96: return launch_cross<96>(p, s);
    case 128: return launch_cross<128>(p, s);
    default: return SAFE_ERR_UNSUPPORTED;
  }
}

bool sizes_ok(int B, int N, int H) {
  return B >= 1 && N >= 1 && H >= 1 && B <= 65535 && H <= 65535 &&
         static_cast<int64_t>(B) * N <= INT_MAX;
}

// Fill the query maps of a cross-attention launch (dense or gathered rows).
safe_status fill_cross(CrossParams& p, const void* Q, const int32_t* q_idx, int nq, const void* Ky, const void* Vy,
                       const int32_t* valid_len, const float* w, void* O, float* partial, int B, int N, int M, int H,
                       int d, float scale) {
  p = CrossParams{};
  for (int c = 0; c < nchunks(d); ++c) {
    if (q_idx == nullptr) {
      if (!encode_rows_map(&p.q_map[c], Q, B, N, H, d, c)) return SAFE_ERR_CUDA;
    } else {
      if (!encode_gather_map(&p.qg_map[c], Q, B, N, H, d, c)) return SAFE_ERR_CUDA;
    }
  }
  if (O != nullptr)
    for (int c = 0; c < nchunks(d); ++c)
      if (!encode_rows_map(&p.o_map[c], O, B, nq, H, d, c)) return SAFE_ERR_CUDA;
  p.Ky = static_cast<const __nv_bfloat16*>(Ky);
  p.Vy = static_cast<const __nv_bfloat16*>(Vy);
  p.valid_len = valid_len;
  p.q_idx = q_idx;
  p.w = w;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.partial = partial;
  p.B = B;
  p.N = N;
  p.M = M;
  p.H = H;
  p.nq = nq;
  p.scale_log2 = scale * kLog2e;
  p.gather = q_idx != nullptr;
  return SAFE_OK;
}

}  // namespace

// ---------------------------------------------------------------- allocation-free PCSP
// Scratch for safe_pcsp_topk_noalloc: the per-head partial scores [B, H, N]
// live in this fixed array, which every GPU that loads the library keeps
// until the process exits. Host code must not use the name as an address (it
// is only a host-side stand-in); the device address comes from
// cudaGetSymbolAddress, looked up once per device below.
constexpr size_t kNoAllocScratchFloats = size_t(1) << 21;  // 2 Mi floats = 8 MiB
static __device__ __align__(256) float g_pcsp_noalloc_scratch[kNoAllocScratchFloats];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call made with that device current).
safe_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAFE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SAFE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_pcsp_noalloc_scratch) != cudaSuccess || p == nullptr) return SAFE_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return SAFE_OK;
}

// Parameters of an SRSU launch (tensor maps of Q or its gather map and of the
// cache K / V); false when a map cannot be encoded.
bool fill_srsu(FlashParams& p, const void* Q, int q_compact, const int32_t* S, int k, const void* Kc, const void* Vc,
               void* O_S, float* lse, int B, int N, int H, int d, float scale) {
  if (!encode_v_map(&p.v_map, Vc, B, N, H, d)) return false;
  for (int c = 0; c < nchunks(d); ++c) {
    bool ok = encode_rows_map(&p.k_map[c], Kc, B, N, H, d, c);
    ok = ok && (q_compact ? encode_rows_map(&p.q_map[c], Q, B, k, H, d, c)
                          : encode_gather_map(&p.qg_map[c], Q, B, N, H, d, c));
    ok = ok && encode_rows_map(&p.o_map[c], O_S, B, k, H, d, c);
    if (!ok) return false;
  }
  p.S = S;
  p.O = static_cast<__nv_bfloat16*>(O_S);
  p.lse = lse;
  p.B = B;
  p.N = N;
  p.H = H;
  p.n_q = k;
  p.scale_log2 = scale * kLog2e;
  p.gather = q_compact ? 0 : 1;
  return true;
}

// With the query rows gathered from a full-size Q and room for them in the
// workspace (safe_srsu_workspace_bytes): copy the rows of S into the end of
// the workspace as a compact [B, k, H, d] tensor and point Q there, so the
// kernel loads each query tile by one tiled copy instead of per-row gathers;
// the rest of the workspace is left for the key split. False on a launch
// error.
bool srsu_compact_q(const void*& Q, int& q_compact, const int32_t* S, int k, int B, int N, int H, int d, void* ws,
                    size_t& ws_bytes, cudaStream_t s) {
  if (q_compact || ws == nullptr || !aligned16(ws)) return true;
  const size_t split = align256(safe_attn_workspace_bytes(B, k, N, H, d));
  const size_t need = split + static_cast<size_t>(B) * k * H * d * 2;
  if (ws_bytes < need) return true;
  const long long rows = static_cast<long long>(B) * k;
  if ((rows + 7) / 8 > INT_MAX) return true;
  void* qc = static_cast<uint8_t*>(ws) + split;
  gather_rows_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, s>>>(static_cast<const uint4*>(Q), S,
                                                                           static_cast<uint4*>(qc), B, N, k,
                                                                           H * d / 8);
  if (cudaGetLastError() != cudaSuccess) return false;
  Q = qc;
  q_compact = 1;
  ws_bytes = split;
  return true;
}

}  // namespace

extern "C" {

int safe_abi_version(void) { return kAbiVersion; }

const char* safe_status_string(int status) {
  switch (status) {
    case SAFE_OK: return "ok";
    case SAFE_ERR_INVALID_ARG: return "invalid argument";
    case SAFE_ERR_UNSUPPORTED: return "unsupported shape";
    case SAFE_ERR_CUDA: return "CUDA error";
    case SAFE_ERR_TIMEOUT: return "device wait timed out";
    case SAFE_ERR_DEVICE_CHECK: return "device-side input check failed";
    default: return "unknown status";
  }
}

safe_status safe_mask_classify(const void* mask, int dtype, const int64_t sizes[4], const int64_t strides[4],
                               int64_t* d_result, void* stream) {
  if (mask == nullptr || sizes == nullptr || strides == nullptr || d_result == nullptr) return SAFE_ERR_INVALID_ARG;
  if (dtype < SAFE_BOOL || dtype > SAFE_BF16) return SAFE_ERR_INVALID_ARG;
  for (int a = 0; a < 4; ++a)
    if (sizes[a] < 1 || strides[a] < 0) return SAFE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_result) & 7u) != 0) return SAFE_ERR_INVALID_ARG;
  const int esize = (dtype <= SAFE_U8) ? 1 : (dtype == SAFE_F32 ? 4 : 2);
  if ((reinterpret_cast<uintptr_t>(mask) % esize) != 0) return SAFE_ERR_INVALID_ARG;
  ClassifyParams p{};
  p.mask = static_cast<const uint8_t*>(mask);
  p.dtype = dtype;
  p.esize = esize;
  p.nb = strides[0] == 0 ? 1 : sizes[0];
  p.nh = strides[1] == 0 ? 1 : sizes[1];
  p.nq = strides[2] == 0 ? 1 : sizes[2];
  p.nk = strides[3] == 0 ? 1 : sizes[3];
  p.s0 = strides[0];
  p.s1 = strides[1];
  p.s2 = strides[2];
  p.s3 = strides[3];
  p.nfail = reinterpret_cast<unsigned long long*>(d_result + 1);
  p.first_fail = reinterpret_cast<unsigned long long*>(d_result + 2);
  cudaStream_t s = as_stream(stream);
  classify_init_kernel<<<1, 1, 0, s>>>(d_result);
  const int64_t rows = p.nb * p.nh * p.nq;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (rows + 7) / 8;
  const int grid = static_cast<int>(want < static_cast<int64_t>(sms) * 16 ? want : static_cast<int64_t>(sms) * 16);
  classify_rows_kernel<<<grid, 256, 0, s>>>(p);
  classify_finalize_kernel<<<1, 1, 0, s>>>(d_result);
  return launch_status();
}

safe_status safe_mask_classify_sync(const void* mask, int dtype, const int64_t sizes[4], const int64_t strides[4],
                                    int64_t* d_result, int64_t* h_result, void* stream) {
  if (h_result == nullptr) return SAFE_ERR_INVALID_ARG;
  safe_status st = safe_mask_classify(mask, dtype, sizes, strides, d_result, stream);
  if (st != SAFE_OK) return st;
  cudaStream_t s = as_stream(stream);
  if (cudaMemcpyAsync(h_result, d_result, 3 * sizeof(int64_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return SAFE_ERR_CUDA;
  return cudaStreamSynchronize(s) == cudaSuccess ? SAFE_OK : SAFE_ERR_CUDA;
}

size_t safe_attn_workspace_bytes(int B, int n_q, int N, int H, int d) {
  if (B < 1 || n_q < 1 || N < 1 || H < 1 || !supported_d(d)) return 0;
  return plan_flash(B, H, n_q, N, d, device_sms()).ws_bytes;
}

safe_status safe_attn_self(const void* Q, const void* K, const void* V, void* O, float* lse, int B, int N, int H,
                           int d, float scale, void* ws, size_t ws_bytes, void* stream) {
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SAFE_ERR_INVALID_ARG;
  if (!sizes_ok(B, N, H) || !scale_ok(scale)) return SAFE_ERR_INVALID_ARG;
  if (!supported_d(d)) return SAFE_ERR_UNSUPPORTED;
  FlashParams p{};
  for (int c = 0; c < nchunks(d); ++c) {
    if (!encode_rows_map(&p.q_map[c], Q, B, N, H, d, c) || !encode_rows_map(&p.k_map[c], K, B, N, H, d, c) ||
        !encode_rows_map(&p.o_map[c], O, B, N, H, d, c))
      return SAFE_ERR_CUDA;
  }
  if (!encode_v_map(&p.v_map, V, B, N, H, d)) return SAFE_ERR_CUDA;
  p.S = nullptr;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.lse = lse;
  p.B = B;
  p.N = N;
  p.H = H;
  p.n_q = N;
  p.scale_log2 = scale * kLog2e;
  p.gather = 0;
  return dispatch_flash(d, p, ws, ws_bytes, as_stream(stream));
}

size_t safe_srsu_workspace_bytes(int B, int k, int N, int H, int d) {
  if (B < 1 || k < 1 || N < 1 || H < 1 || !supported_d(d)) return 0;
  return align256(safe_attn_workspace_bytes(B, k, N, H, d)) + static_cast<size_t>(B) * k * H * d * 2;
}

safe_status safe_srsu_attn(const void* Q, int q_compact, const int32_t* S, int k, const void* Kc, const void* Vc,
                           void* O_S, float* lse, int B, int N, int H, int d, float scale, void* ws, size_t ws_bytes,
                           void* stream) {
  if (!aligned16(Q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(O_S)) return SAFE_ERR_INVALID_ARG;
  if (!sizes_ok(B, N, H) || k < 1 || k > N || !scale_ok(scale)) return SAFE_ERR_INVALID_ARG;
  if (!q_compact && S == nullptr) return SAFE_ERR_INVALID_ARG;
  if (!supported_d(d)) return SAFE_ERR_UNSUPPORTED;
  if (!srsu_compact_q(Q, q_compact, S, k, B, N, H, d, ws, ws_bytes, as_stream(stream))) return SAFE_ERR_CUDA;
  FlashParams p{};
  if (!fill_srsu(p, Q, q_compact, S, k, Kc, Vc, O_S, lse, B, N, H, d, scale)) return SAFE_ERR_CUDA;
  return dispatch_flash(d, p, ws, ws_bytes, as_stream(stream));
}

safe_status safe_srsu_attn_assembled(const void* Q, int q_compact, const int32_t* S, int k, const void* Kcur,
                                     const void* Vcur, int cur_compact, const void* Kc, const void* Vc, void* O_S,
                                     float* lse, int B, int N, int H, int d, float scale, void* ws, size_t ws_bytes,
                                     void* stream) {
  if (!aligned16(Q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(O_S) || !aligned16(Kcur) ||
      !aligned16(Vcur) || S == nullptr)
    return SAFE_ERR_INVALID_ARG;
  if (!sizes_ok(B, N, H) || k < 1 || k > N || !scale_ok(scale)) return SAFE_ERR_INVALID_ARG;
  if (!supported_d(d)) return SAFE_ERR_UNSUPPORTED;
  if (!srsu_compact_q(Q, q_compact, S, k, B, N, H, d, ws, ws_bytes, as_stream(stream))) return SAFE_ERR_CUDA;
  FlashParams p{};
  if (!fill_srsu(p, Q, q_compact, S, k, Kc, Vc, O_S, lse, B, N, H, d, scale)) return SAFE_ERR_CUDA;
  p.k_cur = static_cast<const __nv_bfloat16*>(Kcur);
  p.v_cur = static_cast<const __nv_bfloat16*>(Vcur);
  p.cur_compact = cur_compact ? 1 : 0;
  return dispatch_flash(d, p, ws, ws_bytes, as_stream(stream), true);
}

safe_status safe_attn_cross(const void* Q, const int32_t* q_idx, int nq, const void* Ky, const void* Vy,
                            const int32_t* valid_len, void* O, int B, int N, int M, int H, int d, float scale,
                            void* stream) {
  if (!aligned16(Q) || !aligned16(Ky) || !aligned16(Vy) || !aligned16(O) || valid_len == nullptr)
    return SAFE_ERR_INVALID_ARG;
  if (!sizes_ok(B, N, H) || M < 1 || !scale_ok(scale)) return SAFE_ERR_INVALID_ARG;
  if (q_idx == nullptr ? nq != N : (nq < 1 || nq > N)) return SAFE_ERR_INVALID_ARG;
  if (!supported_d(d) || M > 256) return SAFE_ERR_UNSUPPORTED;
  CrossParams p;
  safe_status st = fill_cross(p, Q, q_idx, nq, Ky, Vy, valid_len, nullptr, O, nullptr, B, N, M, H, d, scale);
  if (st != SAFE_OK) return st;
  return dispatch_cross(d, p, as_stream(stream));
}

size_t safe_pcsp_workspace_bytes(int B, int N, int H) {
  if (B < 1 || N < 1 || H < 1) return 0;
  return static_cast<size_t>(B) * H * N * sizeof(float);
}

safe_status safe_topk_partition(const float* scores, int B, int N, int k, int32_t* S, int32_t* C, void* stream) {
  if (scores == nullptr || S == nullptr || B < 1 || N < 1 || k < 1 || k > N) return SAFE_ERR_INVALID_ARG;
  if (N <= kTopkSmemKeys) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
      attr_err = cudaFuncSetAttribute(topk_partition_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kTopkSmemKeys * static_cast<int>(sizeof(uint32_t)));
    });
    if (attr_err != cudaSuccess) return SAFE_ERR_CUDA;
    topk_partition_kernel<true><<<B, kTopkThreads, N * sizeof(uint32_t), as_stream(stream)>>>(scores, N, k, S, C);
  } else {
    topk_partition_kernel<false><<<B, kTopkThreads, 0, as_stream(stream)>>>(scores, N, k, S, C);
  }
  return launch_status();
}

safe_status safe_pcsp_topk(const void* Q, const void* Ky, const int32_t* valid_len, const float* w, int B, int N,
                           int M, int H, int d, float scale, float* scores, int accumulate, int k, int32_t* S,
                           int32_t* C, void* ws, size_t ws_bytes, void* stream) {
  if (scores == nullptr || !sizes_ok(B, N, H) || k < 0 || k > N) return SAFE_ERR_INVALID_ARG;
  if (k > 0 && S == nullptr) return SAFE_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  if (Q != nullptr) {
    if (!aligned16(Q) || !aligned16(Ky) || valid_len == nullptr || M < 1 || !scale_ok(scale))
      return SAFE_ERR_INVALID_ARG;
    if (!supported_d(d) || M > 256) return SAFE_ERR_UNSUPPORTED;
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 ||
        ws_bytes < safe_pcsp_workspace_bytes(B, N, H))
      return SAFE_ERR_INVALID_ARG;
    CrossParams p;
    // The value operand is not read when only scores are produced (O = null).
    safe_status st = fill_cross(p, Q, nullptr, N, Ky, Ky, valid_len, w, nullptr, static_cast<float*>(ws), B, N, M,
                                H, d, scale);
    if (st != SAFE_OK) return st;
    st = dispatch_cross(d, p, s);
    if (st != SAFE_OK) return st;
    dim3 grid((N + 255) / 256, B);
    pcsp_reduce_kernel<<<grid, 256, 0, s>>>(static_cast<const float*>(ws), scores, B, H, N, accumulate ? 1 : 0);
    st = launch_status();
    if (st != SAFE_OK) return st;
  }
  if (k > 0) return safe_topk_partition(scores, B, N, k, S, C, stream);
  return SAFE_OK;
}

safe_status safe_attn_cross_pcsp(const void* Q, const void* Ky, const void* Vy, const int32_t* valid_len,
                                 const float* w, void* O, int B, int N, int M, int H, int d, float scale,
                                 float* scores, int accumulate, int k, int32_t* S, int32_t* C, void* ws,
                                 size_t ws_bytes, void* stream) {
  if (!aligned16(Q) || !aligned16(Ky) || !aligned16(Vy) || !aligned16(O) || valid_len == nullptr || scores == nullptr)
    return SAFE_ERR_INVALID_ARG;
  if (!sizes_ok(B, N, H) || M < 1 || !scale_ok(scale) || k < 0 || k > N || (k > 0 && S == nullptr))
    return SAFE_ERR_INVALID_ARG;
  if (!supported_d(d) || M > 256) return SAFE_ERR_UNSUPPORTED;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < safe_pcsp_workspace_bytes(B, N, H))
    return SAFE_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  CrossParams p;
  // one pass over the queries: the output rows and, from the same
  // probabilities, the per-head score partials
  safe_status st = fill_cross(p, Q, nullptr, N, Ky, Vy, valid_len, w, O, static_cast<float*>(ws), B, N, M, H, d,
                              scale);
  if (st != SAFE_OK) return st;
  st = dispatch_cross(d, p, s);
  if (st != SAFE_OK) return st;
  pcsp_reduce_kernel<<<dim3((N + 255) / 256, B), 256, 0, s>>>(static_cast<const float*>(ws), scores, B, H, N,
                                                              accumulate ? 1 : 0);
  st = launch_status();
  if (st != SAFE_OK) return st;
  if (k > 0) return safe_topk_partition(scores, B, N, k, S, C, stream);
  return SAFE_OK;
}

safe_status safe_pcsp_topk_noalloc(const void* Q, const void* Ky, const int32_t* valid_len, const float* w, int B,
                                   int N, int M, int H, int d, float scale, float* scores, int accumulate, int k,
                                   int32_t* S, int32_t* C, void* stream) {
  void* ws = nullptr;
  size_t ws_bytes = 0;
  if (Q != nullptr) {
    if (B < 1 || N < 1 || H < 1) return SAFE_ERR_INVALID_ARG;
    const size_t need = safe_pcsp_workspace_bytes(B, N, H);
    if (need > sizeof(g_pcsp_noalloc_scratch)) return SAFE_ERR_UNSUPPORTED;  // B*H*N above 2^21
    const safe_status st = noalloc_scratch(&ws);
    if (st != SAFE_OK) return st;
    ws_bytes = sizeof(g_pcsp_noalloc_scratch);
  }
  // Every element of the [B, H, N] partial block is written by the scoring
  // kernel before the head sum reads it, so nothing needs clearing.
  return safe_pcsp_topk(Q, Ky, valid_len, w, B, N, M, H, d, scale, scores, accumulate, k, S, C, ws, ws_bytes,
                        stream);
}

safe_status safe_ctx_cache_scatter(const void* Ksrc, const void* Vsrc, int src_compact, const int32_t* S, int k,
                                   void* Kc, void* Vc, int B, int N, int H, int d, void* stream) {
  if (!aligned16(Ksrc) || !aligned16(Vsrc) || !aligned16(Kc) || !aligned16(Vc)) return SAFE_ERR_INVALID_ARG;
  if (!sizes_ok(B, N, H) || d < 8 || (d % 8) != 0) return SAFE_ERR_INVALID_ARG;
  if (S != nullptr && (k < 1 || k > N)) return SAFE_ERR_INVALID_ARG;
  if (S == nullptr && src_compact) return SAFE_ERR_INVALID_ARG;
  const int row_units = H * d * 2 / 16;
  const int64_t rows = S != nullptr ? static_cast<int64_t>(B) * k : static_cast<int64_t>(B) * N;
  const int64_t blocks = (rows * 32 + 255) / 256;
  if (blocks > INT_MAX) return SAFE_ERR_UNSUPPORTED;
  cache_scatter_kernel<<<static_cast<unsigned>(blocks), 256, 0, as_stream(stream)>>>(
      static_cast<const uint4*>(Ksrc), static_cast<const uint4*>(Vsrc), src_compact, S, k, static_cast<uint4*>(Kc),
      static_cast<uint4*>(Vc), B, N, row_units);
  return launch_status();
}

// ---------------------------------------------------------------- sensitivity field and SW-CFG
size_t safe_sensitivity_workspace_bytes(int B, int N) {
  if (B < 1 || N < 1) return 0;
  return align256(static_cast<size_t>(B) * N * sizeof(float)) + align256(static_cast<size_t>(B) * 2 * sizeof(uint32_t));
}

safe_status safe_sensitivity_field(const float* scores, float* s, int B, int grid_h, int grid_w, float sigma,
                                   float truncate, void* ws, size_t ws_bytes, void* stream) {
  if (scores == nullptr || s == nullptr || scores == s || B < 1 || B > 65535 || grid_h < 1 || grid_w < 1)
    return SAFE_ERR_INVALID_ARG;
  if (static_cast<int64_t>(grid_h) * grid_w > INT_MAX / 2) return SAFE_ERR_INVALID_ARG;
  if (!std::isfinite(sigma) || sigma < 0.f || !std::isfinite(truncate) || truncate <= 0.f) return SAFE_ERR_INVALID_ARG;
  const int N = grid_h * grid_w;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < safe_sensitivity_workspace_bytes(B, N))
    return SAFE_ERR_INVALID_ARG;
  SmoothParams p{};
  // the taps of G_sigma, in double, then rounded to fp32
  const double r_real = sigma > 0.f ? std::floor(static_cast<double>(truncate) * sigma + 0.5) : 0.0;
  if (r_real > kMaxSmoothRadius) return SAFE_ERR_UNSUPPORTED;
  p.r = static_cast<int>(r_real);
  if (p.r == 0) {
    p.taps[0] = 1.f;
  } else {
    double g[kMaxTaps], sum = 0.0;
    for (int t = -p.r; t <= p.r; ++t) {
      g[t + p.r] = std::exp(-(static_cast<double>(t) * t) / (2.0 * sigma * sigma));
      sum += g[t + p.r];
    }
    for (int t = 0; t <= 2 * p.r; ++t) p.taps[t] = static_cast<float>(g[t] / sum);
  }
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.in = scores;
  p.rows = reinterpret_cast<float*>(w);
  p.out = s;
  p.minmax = reinterpret_cast<uint32_t*>(w + align256(static_cast<size_t>(B) * N * sizeof(float)));
  p.B = B;
  p.gh = grid_h;
  p.gw = grid_w;
  cudaStream_t st = as_stream(stream);
  const dim3 grid((N + 255) / 256, B);
  smooth_rows_kernel<<<grid, 256, 0, st>>>(p);
  smooth_cols_kernel<<<grid, 256, 0, st>>>(p);
  norm01_kernel<<<grid, 256, 0, st>>>(s, p.minmax, N);
  return launch_status();
}

// ---------------------------------------------------------------- row-wise layers of the block
size_t safe_gather_linear_workspace_bytes(int B, int k, int d_in) {
  if (B < 1 || k < 1 || d_in < 1) return 0;
  return static_cast<size_t>(B) * k * d_in * 2;
}

safe_status safe_gather_linear(const void* X, const int32_t* S, int k, const void* Wt, const float* bias, int act,
                               void* Y, int B, int N, int d_in, int d_out, void* ws, size_t ws_bytes, void* stream) {
  if (!aligned16(X) || !aligned16(Wt) || !aligned16(Y)) return SAFE_ERR_INVALID_ARG;
  if (bias != nullptr && (reinterpret_cast<uintptr_t>(bias) & 3u) != 0) return SAFE_ERR_INVALID_ARG;
  if (!sizes_ok(B, N, 1) || (S != nullptr && (k < 1 || k > N))) return SAFE_ERR_INVALID_ARG;
  if (d_in < 64 || d_in % 8 != 0 || d_out < 8 || d_out % 8 != 0 || (act != 0 && act != 1)) return SAFE_ERR_INVALID_ARG;
  if (S != nullptr && aligned16(ws) && ws_bytes >= safe_gather_linear_workspace_bytes(B, k, d_in)) {
    // the rows of S as a compact [B, k, d_in] matrix, then the GEMM over
    // every row of it (tiled operand copies instead of per-row gathers)
    const long long rows = static_cast<long long>(B) * k;
    if ((rows + 7) / 8 > INT_MAX) return SAFE_ERR_UNSUPPORTED;
    gather_rows_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, as_stream(stream)>>>(
        static_cast<const uint4*>(X), S, static_cast<uint4*>(ws), B, N, k, d_in / 8);
    if (cudaGetLastError() != cudaSuccess) return SAFE_ERR_CUDA;
    X = ws;
    N = k;
    S = nullptr;
  }
  const int R = S != nullptr ? k : N;
  // plain rows: CTA pairs on 256 x 256 tiles; rows of S gathered in the
  // kernel (no workspace): one CTA per 128 x 256 tile
  const bool pairs = S == nullptr;
  const int64_t m_tiles = (R + (pairs ? 255 : 127)) / (pairs ? 256 : 128), n_tiles = (d_out + 255) / 256;
  const int64_t tiles = static_cast<int64_t>(B) * m_tiles * n_tiles;
  if (tiles > INT_MAX) return SAFE_ERR_UNSUPPORTED;
  LinearParams p{};
  if (!encode_matrix_map(&p.x_map, X, static_cast<uint64_t>(d_in), static_cast<uint64_t>(B) * N, 64, 1) ||
      !encode_matrix_map(&p.xt_map, X, static_cast<uint64_t>(d_in), static_cast<uint64_t>(B) * N, 64, 128) ||
      !encode_matrix_map(&p.w_map, Wt, static_cast<uint64_t>(d_in), static_cast<uint64_t>(d_out), 64, 256) ||
      !encode_matrix_map(&p.w2_map, Wt, static_cast<uint64_t>(d_in), static_cast<uint64_t>(d_out), 64, 128))
    return SAFE_ERR_CUDA;
  p.S = S;
  p.bias = bias;
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.B = B;
  p.N = N;
  p.R = R;
  p.d_in = d_in;
  p.d_out = d_out;
  p.act = act;
  p.m_tiles = static_cast<int>(m_tiles);
  p.n_tiles = static_cast<int>(n_tiles);
  p.tiles = static_cast<int>(tiles);
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(linear_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kLinSmem);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(linear_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kLin2Smem);
  });
  if (attr_err != cudaSuccess) return SAFE_ERR_CUDA;
  const int sms = device_sms();
  if (pairs) {
    // as many pairs as can be resident at once (a GPC with an odd number of
    // free SMs leaves one of them out), so that every pair starts at once
    static int max_pairs[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    int& mp = max_pairs[dev >= 0 && dev < 64 ? dev : 0];
    if (mp == 0) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(2 * (sms / 2)));
      cfg.blockDim = dim3(kLinThreads);
      cfg.dynamicSmemBytes = kLin2Smem;
      int n = 0;
      mp = cudaOccupancyMaxActiveClusters(&n, linear_pair_kernel, &cfg) == cudaSuccess && n > 0 ? n : sms / 2;
    }
    const int n_pairs = static_cast<int>(tiles < mp ? tiles : mp);
    linear_pair_kernel<<<2 * (n_pairs > 0 ? n_pairs : 1), kLinThreads, kLin2Smem, as_stream(stream)>>>(p);
  } else {
    const int grid = static_cast<int>(tiles < sms ? tiles : sms);
    linear_kernel<<<grid, kLinThreads, kLinSmem, as_stream(stream)>>>(p);
  }
  return launch_status();
}

safe_status safe_partition_indicator(const int32_t* S, int k, float* s, int B, int N, void* stream) {
  if (S == nullptr || s == nullptr || B < 1 || B > 65535 || N < 1 || k < 1 || k > N) return SAFE_ERR_INVALID_ARG;
  partition_indicator_kernel<<<dim3((N + 255) / 256, B), 256, 0, as_stream(stream)>>>(S, k, s, N);
  return launch_status();
}

safe_status safe_sw_cfg(const void* f_c, const void* f_u, const float* s, void* out, int dtype, int B, int N, int C,
                        float gamma_ctx, float gamma_sens, void* stream) {
  if (f_c == nullptr || f_u == nullptr || s == nullptr || out == nullptr || B < 1 || N < 1 || C < 1)
    return SAFE_ERR_INVALID_ARG;
  if (dtype != SAFE_F32 && dtype != SAFE_BF16) return SAFE_ERR_UNSUPPORTED;
  if (!std::isfinite(gamma_ctx) || !std::isfinite(gamma_sens)) return SAFE_ERR_INVALID_ARG;
  const size_t esize = dtype == SAFE_F32 ? 4 : 2;
  auto aligned = [](const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; };
  if (!aligned(f_c, esize) || !aligned(f_u, esize) || !aligned(out, esize) || !aligned(s, 4))
    return SAFE_ERR_INVALID_ARG;
  const size_t total = static_cast<size_t>(B) * N * C;
  const int vec = static_cast<int>(16 / esize);
  const bool vec_ok = (C % vec) == 0 && aligned(f_c, 16) && aligned(f_u, 16) && aligned(out, 16);
  const size_t n_vec = vec_ok ? total / vec : total;
  const size_t want = (n_vec + 255) / 256;
  const unsigned blocks = static_cast<unsigned>(want < static_cast<size_t>(device_sms()) * 16 ? (want ? want : 1)
                                                                                          : static_cast<size_t>(device_sms()) * 16);
  const float diff = gamma_sens - gamma_ctx;
  cudaStream_t st = as_stream(stream);
  if (dtype == SAFE_F32) {
    auto fc = static_cast<const float*>(f_c);
    auto fu = static_cast<const float*>(f_u);
    auto o = static_cast<float*>(out);
    if (vec_ok) sw_cfg_kernel<float, 4><<<blocks, 256, 0, st>>>(fc, fu, s, o, n_vec, C, gamma_ctx, diff);
    else sw_cfg_kernel<float, 1><<<blocks, 256, 0, st>>>(fc, fu, s, o, n_vec, C, gamma_ctx, diff);
  } else {
    auto fc = static_cast<const __nv_bfloat16*>(f_c);
    auto fu = static_cast<const __nv_bfloat16*>(f_u);
    auto o = static_cast<__nv_bfloat16*>(out);
    if (vec_ok) sw_cfg_kernel<__nv_bfloat16, 8><<<blocks, 256, 0, st>>>(fc, fu, s, o, n_vec, C, gamma_ctx, diff);
    else sw_cfg_kernel<__nv_bfloat16, 1><<<blocks, 256, 0, st>>>(fc, fu, s, o, n_vec, C, gamma_ctx, diff);
  }
  return launch_status();
}

safe_status safe_get_device_status(int* h_status, void* stream) {
  if (h_status == nullptr) return SAFE_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return SAFE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return SAFE_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return SAFE_ERR_CUDA;
  *h_status = v;
  return SAFE_OK;
}

safe_status safe_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 1000000000ull) return SAFE_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(limit_ns);
  return launch_status();
}

}  // extern "C"
