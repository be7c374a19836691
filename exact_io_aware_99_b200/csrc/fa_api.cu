// fa_api.cu -- the C ABI declared in include/fa.h: argument checks, TMA
// tensor-map encoding, workspace carving and kernel launches.  No device
// memory is allocated here; the only device state is the status word below.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "fa_fp8.h"
#include "fa_internal.h"

namespace {

// Written by a kernel whose bounded wait ran out (first site wins).
__device__ int g_fa_status = 0;

constexpr unsigned long long kDefaultLimitNs = 2000000000ull;
std::atomic<unsigned long long> g_limit_ns{kDefaultLimitNs};
// Key-tile size of the dense bf16 forward: 0 = the built-in table, else 64
// or 128 (fa_set_forward_key_tile).
std::atomic<int> g_fwd_key_tile{0};

// Key-tile size of the dense bf16 forward for a problem: the 64-key kernel
// (two score buffers per query tile) or the 128-key kernel.  The table is the
// measured winner on B200 (both kernels timed on the same inputs, L2 flushed,
// B H N = 262144): the 64-key kernel is ahead only for short causal problems,
// where most key steps are diagonal or ragged and its finer key tiles skip
// more masked work (d = 128 causal: +4 % at N = 128 and 256, even at 512;
// d = 64 causal: +6 % at N = 512); elsewhere its twice as many, half as wide
// score MMAs cost 6-25 %.
int forward_key_tile(int d, int N, int causal) {
  const int forced = g_fwd_key_tile.load(std::memory_order_relaxed);
  if (forced == 64 || forced == 128) return forced;
  if (!causal) return 128;
  return N <= (d == 128 ? 256 : 512) ? 64 : 128;
}
thread_local int g_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
// Filled in once per device under g_dev_mu; `checked` is published with a
// release store after `status`, so a thread that reads it with acquire and
// sees 1 also sees the status address.
struct DeviceInfo {
  std::atomic<int> checked{0};  // 0 unknown, 1 supported, -1 unsupported
  int* status = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

fa_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return FA_ERR_CUDA;
}

// Checks that the current device is an sm_100 part and returns its launch
// context (status-word address, time limit).
fa_status device_context(void* stream, fa::Launch* L) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  DeviceInfo& di = g_dev[dev];
  int checked = di.checked.load(std::memory_order_acquire);
  if (checked == 0) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    checked = di.checked.load(std::memory_order_relaxed);
    if (checked == 0) {
      cudaDeviceProp prop;
      e = cudaGetDeviceProperties(&prop, dev);
      if (e != cudaSuccess) return cuda_fail(e);
      if (prop.major != 10 || prop.minor != 0) {
        checked = -1;
      } else {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_fa_status);
        if (e != cudaSuccess) return cuda_fail(e);
        di.status = static_cast<int*>(p);
        checked = 1;
      }
      di.checked.store(checked, std::memory_order_release);
    }
  }
  if (checked < 0) return FA_ERR_UNSUPPORTED;
  L->stream = static_cast<cudaStream_t>(stream);
  L->status = di.status;
  L->limit_ns = g_limit_ns.load(std::memory_order_relaxed);
  return FA_OK;
}

fa_status get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode ? FA_OK : FA_ERR_CUDA;
}

// [BH, N, d] bf16 viewed as 3-D {d, N, BH}; box {64, box_rows, 1}; 128-byte
// swizzle; out-of-range rows and columns read as zero (loads) or are not
// written (stores).
fa_status make_map(CUtensorMap* m, const void* base, int BH, int N, int d, int box_rows = 128) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_cuda_error = static_cast<int>(r);
    return FA_ERR_CUDA;
  }
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status check_common(int B, int H, int N, int d, float scale, fa_dtype dtype) {
  if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
  const long long bh = static_cast<long long>(B) * H;
  if (bh > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  if (dtype == FA_BF16) {
    if (d != 64 && d != 80 && d != 128) return FA_ERR_UNSUPPORTED;
    if ((N + 127) / 128 > 65535) return FA_ERR_UNSUPPORTED;  // grid.y limit
    if (static_cast<long long>(N) * d * 2 * bh >= (1LL << 40)) return FA_ERR_UNSUPPORTED;
  } else if (dtype == FA_FP32) {
    if (d < 1 || d > 128) return FA_ERR_UNSUPPORTED;
    if ((N + 63) / 64 > 65535) return FA_ERR_UNSUPPORTED;
  } else {
    return FA_ERR_UNSUPPORTED;
  }
  return FA_OK;
}

struct WsLayout {
  size_t dvec_off, lse2_off, total;
};

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

WsLayout ws_layout(int B, int H, int N, int d) {
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t np = static_cast<size_t>(fa::round_up(N, fa::kTileRows));
  (void)N;
  (void)d;
  WsLayout w;
  w.dvec_off = 0;
  w.lse2_off = up256(bh * np * sizeof(float));
  w.total = w.lse2_off + up256(bh * np * sizeof(float));
  return w;
}

}  // namespace

extern "C" {

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case FA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case FA_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case FA_ERR_CUDA: return "CUDA call failed";
    case FA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

int fa_last_cuda_error(void) { return g_last_cuda_error; }

void fa_set_wait_timeout_ns(unsigned long long ns) {
  g_limit_ns.store(ns ? ns : kDefaultLimitNs, std::memory_order_relaxed);
}

fa_status fa_set_forward_key_tile(int keys) {
  if (keys != 0 && keys != 64 && keys != 128) return FA_ERR_INVALID_ARG;
  g_fwd_key_tile.store(keys, std::memory_order_relaxed);
  return FA_OK;
}

int fa_forward_key_tile(int d, int N, int causal) {
  if (N < 1 || (d != 64 && d != 80 && d != 128)) return 0;
  return forward_key_tile(d, N, causal ? 1 : 0);
}

fa_status fa_device_status(int reset, int* site) {
  fa::Launch L;
  fa_status st = device_context(nullptr, &L);
  if (st != FA_OK) return st;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e);
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_fa_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  if (reset && v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_fa_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e);
  }
  if (site) *site = v;
  return v ? FA_ERR_DEVICE_TIMEOUT : FA_OK;
}

fa_status fa_selftest_wait_timeout(void* stream) {
  fa::Launch L;
  fa_status st = device_context(stream, &L);
  if (st != FA_OK) return st;
  cudaError_t e = fa::launch_selftest_wait(L);
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

fa_status fa_forward_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int H, int N, int d, float scale, int causal, fa_dtype dtype,
                        void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  fa_status st = check_common(B, H, N, d, scale, dtype);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_MISALIGNED;
  fa::Launch L;
  st = device_context(stream, &L);
  if (st != FA_OK) return st;
  const int BH = B * H;
  const int cz = causal ? 1 : 0;
  cudaError_t e;
  if (dtype == FA_FP32) {
    e = fa::launch_fwd_f32(static_cast<const float*>(q), static_cast<const float*>(k),
                           static_cast<const float*>(v), static_cast<float*>(o), lse, BH, N, d,
                           scale, cz, L);
  } else {
    st = get_encoder();
    if (st != FA_OK) return st;
    const int kt = forward_key_tile(d, N, cz);
    CUtensorMap tq, tk, tv, to;
    if ((st = make_map(&tq, q, BH, N, d)) != FA_OK) return st;
    if ((st = make_map(&tk, k, BH, N, d, kt)) != FA_OK) return st;
    if ((st = make_map(&tv, v, BH, N, d, kt)) != FA_OK) return st;
    if ((st = make_map(&to, o, BH, N, d, fa::kStoreBoxRows)) != FA_OK) return st;
    e = kt == 64 ? fa::launch_fwd64_sm100(tq, tk, tv, to, lse, BH, N, d, scale, cz, L)
                 : fa::launch_fwd_sm100(tq, tk, tv, to, o, lse, BH, N, d, scale, cz, nullptr, L);
  }
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

fa_status fa_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int N, int d, float scale, int causal, void* stream) {
  return fa_forward_ex(q, k, v, o, lse, B, H, N, d, scale, causal, FA_BF16, stream);
}

fa_status fa_forward_blocksparse(const void* q, const void* k, const void* v, void* o,
                                 float* lse, int B, int H, int N, int d, float scale, int causal,
                                 const unsigned char* block_mask, int mask_heads, void* stream) {
  if (!q || !k || !v || !o || !lse || !block_mask) return FA_ERR_INVALID_ARG;
  fa_status st = check_common(B, H, N, d, scale, FA_BF16);
  if (st != FA_OK) return st;
  if (mask_heads != 1 && mask_heads != H) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_MISALIGNED;
  fa::Launch L;
  st = device_context(stream, &L);
  if (st != FA_OK) return st;
  const int BH = B * H;
  st = get_encoder();
  if (st != FA_OK) return st;
  CUtensorMap tq, tk, tv, to;
  if ((st = make_map(&tq, q, BH, N, d)) != FA_OK) return st;
  if ((st = make_map(&tk, k, BH, N, d)) != FA_OK) return st;
  if ((st = make_map(&tv, v, BH, N, d)) != FA_OK) return st;
  if ((st = make_map(&to, o, BH, N, d, fa::kStoreBoxRows)) != FA_OK) return st;
  const fa::BlockMaskArg bm{block_mask, mask_heads, H};
  cudaError_t e =
      fa::launch_fwd_sm100(tq, tk, tv, to, o, lse, BH, N, d, scale, causal ? 1 : 0, &bm, L);
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

size_t fa_backward_workspace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || d < 1 || d > 128) return 0;
  return ws_layout(B, H, N, d).total;
}

fa_status fa_backward_ex(const void* q, const void* k, const void* v, const void* o,
                         const void* dO, const float* lse, void* dq, void* dk, void* dv, int B,
                         int H, int N, int d, float scale, int causal, void* workspace,
                         size_t workspace_bytes, fa_dtype dtype, void* stream) {
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  fa_status st = check_common(B, H, N, d, scale, dtype);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) ||
      !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_MISALIGNED;
  const WsLayout w = ws_layout(B, H, N, d);
  if (!workspace || workspace_bytes < w.total ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FA_ERR_WORKSPACE;
  fa::Launch L;
  st = device_context(stream, &L);
  if (st != FA_OK) return st;
  const int BH = B * H;
  const int cz = causal ? 1 : 0;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* dvec = reinterpret_cast<float*>(ws + w.dvec_off);
  float* lse2 = reinterpret_cast<float*>(ws + w.lse2_off);
  cudaError_t e;
  if (dtype == FA_FP32) {
    e = fa::launch_bwd_preprocess(o, dO, lse, dvec, nullptr, BH, N, d, 0, L);
    if (e != cudaSuccess) return cuda_fail(e);
    e = fa::launch_bwd_f32(static_cast<const float*>(q), static_cast<const float*>(k),
                           static_cast<const float*>(v), static_cast<const float*>(dO), lse, dvec,
                           static_cast<float*>(dq), static_cast<float*>(dk),
                           static_cast<float*>(dv), BH, N, d, scale, cz, L);
    return e == cudaSuccess ? FA_OK : cuda_fail(e);
  }
  st = get_encoder();
  if (st != FA_OK) return st;
  CUtensorMap tq, tk, tv, tdo;
  if ((st = make_map(&tq, q, BH, N, d)) != FA_OK) return st;
  if ((st = make_map(&tk, k, BH, N, d)) != FA_OK) return st;
  if ((st = make_map(&tv, v, BH, N, d)) != FA_OK) return st;
  if ((st = make_map(&tdo, dO, BH, N, d)) != FA_OK) return st;
  e = fa::launch_bwd_sm100(tq, tk, tv, tdo, o, dO, lse, dvec, lse2, dq, dk, dv, BH, N, d, scale,
                           cz, nullptr, L);
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

fa_status fa_backward_blocksparse(const void* q, const void* k, const void* v, const void* o,
                                  const void* dO, const float* lse, void* dq, void* dk, void* dv,
                                  int B, int H, int N, int d, float scale, int causal,
                                  const unsigned char* block_mask, int mask_heads,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv || !block_mask)
    return FA_ERR_INVALID_ARG;
  fa_status st = check_common(B, H, N, d, scale, FA_BF16);
  if (st != FA_OK) return st;
  if (mask_heads != 1 && mask_heads != H) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) ||
      !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_MISALIGNED;
  const WsLayout w = ws_layout(B, H, N, d);
  if (!workspace || workspace_bytes < w.total ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FA_ERR_WORKSPACE;
  fa::Launch L;
  st = device_context(stream, &L);
  if (st != FA_OK) return st;
  const int BH = B * H;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* dvec = reinterpret_cast<float*>(ws + w.dvec_off);
  float* lse2 = reinterpret_cast<float*>(ws + w.lse2_off);
  st = get_encoder();
  if (st != FA_OK) return st;
  CUtensorMap tq, tk, tv, tdo;
  if ((st = make_map(&tq, q, BH, N, d)) != FA_OK) return st;
  if ((st = make_map(&tk, k, BH, N, d)) != FA_OK) return st;
  if ((st = make_map(&tv, v, BH, N, d)) != FA_OK) return st;
  if ((st = make_map(&tdo, dO, BH, N, d)) != FA_OK) return st;
  const fa::BlockMaskArg bm{block_mask, mask_heads, H};
  cudaError_t e = fa::launch_bwd_sm100(tq, tk, tv, tdo, o, dO, lse, dvec, lse2, dq, dk, dv, BH, N,
                                       d, scale, causal ? 1 : 0, &bm, L);
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

// Split-KV partition: the N_k keys' tiles split into ranges of kt_per tiles
// (the last range may be shorter; none is empty).
struct SplitPlan {
  int n_split, kt_per;
};
SplitPlan split_plan(int Nk, int num_splits) {
  const int n_kt = (Nk + 127) / 128;
  int s = num_splits < 1 ? 1 : (num_splits > n_kt ? n_kt : num_splits);
  const int kt_per = (n_kt + s - 1) / s;
  s = (n_kt + kt_per - 1) / kt_per;
  return {s, kt_per};
}

struct SplitWs {
  size_t lse_off, total;
};
SplitWs splitkv_ws(int B, int H, int Nq, int d, int n_split) {
  const size_t rows = static_cast<size_t>(n_split) * B * H * Nq;
  const size_t o_bytes = up256(rows * d * sizeof(float));
  return {o_bytes, o_bytes + up256(rows * sizeof(float))};
}

int fa_splitkv_default_splits(int B, int H, int Nq, int Nk) {
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return 0;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long items = static_cast<long long>(B) * H * (((Nq + 127) / 128 + 1) / 2);
  // Enough splits to give every SM about one item, no more.  A decode item is
  // one query tile streaming its key range, and its rate is set by the
  // softmax -> MMA chain of that tile, not by HBM; further splits only add
  // partials (4 N_q d bytes each) for the combine kernel and a ragged last
  // wave.  Measured on B200 (8 x 16 heads, 128 queries, 16384 keys, d 128):
  // 1 split 4723 GB/s, 2: 4590, 3: 4462, 4: 4427, 6: 4235, 8: 4558.
  const long long want = sms / (items > 0 ? items : 1);
  const int n_kt = (Nk + 127) / 128;
  const int s = static_cast<int>(want < 1 ? 1 : (want > n_kt ? n_kt : want));
  return split_plan(Nk, s).n_split;
}

size_t fa_splitkv_workspace_size(int B, int H, int Nq, int Nk, int d, int num_splits) {
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || d < 1 || d > 128 || num_splits < 1) return 0;
  return splitkv_ws(B, H, Nq, d, split_plan(Nk, num_splits).n_split).total;
}

fa_status fa_forward_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int H, int Nq, int Nk, int d, float scale, int causal,
                             int num_splits, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (!q || !k || !v || !o || !lse || num_splits < 1) return FA_ERR_INVALID_ARG;
  fa_status st = check_common(B, H, Nq, d, scale, FA_BF16);
  if (st != FA_OK) return st;
  st = check_common(B, H, Nk, d, scale, FA_BF16);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_MISALIGNED;
  if (static_cast<long long>(B) * H * Nq > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  const SplitPlan sp = split_plan(Nk, num_splits);
  const SplitWs w = splitkv_ws(B, H, Nq, d, sp.n_split);
  if (!workspace || workspace_bytes < w.total ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return FA_ERR_WORKSPACE;
  fa::Launch L;
  st = device_context(stream, &L);
  if (st != FA_OK) return st;
  const int BH = B * H;
  st = get_encoder();
  if (st != FA_OK) return st;
  CUtensorMap tq, tk, tv;
  if ((st = make_map(&tq, q, BH, Nq, d)) != FA_OK) return st;
  if ((st = make_map(&tk, k, BH, Nk, d)) != FA_OK) return st;
  if ((st = make_map(&tv, v, BH, Nk, d)) != FA_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const fa::SplitKv sk{Nk, Nk - Nq, sp.n_split, sp.kt_per, reinterpret_cast<float*>(ws),
                       reinterpret_cast<float*>(ws + w.lse_off)};
  cudaError_t e = fa::launch_fwd_splitkv_sm100(tq, tk, tv, BH, Nq, d, scale, causal ? 1 : 0, sk, L);
  if (e != cudaSuccess) return cuda_fail(e);
  e = fa::launch_splitkv_combine(sk.part_o, sk.part_lse, o, lse, sp.n_split, BH * Nq, d, L);
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

fa_status fa_backward(const void* q, const void* k, const void* v, const void* o, const void* dO,
                      const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                      float scale, int causal, void* workspace, size_t workspace_bytes,
                      void* stream) {
  return fa_backward_ex(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, workspace,
                        workspace_bytes, FA_BF16, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free backward.
//
// The ordinary backward needs a caller-provided workspace.  Some callers have
// no way to provide one: code running where every byte of device memory is
// owned by some other allocator it cannot reach, plugins and callbacks that
// are handed tensors but no means to reserve device memory, and
// latency-bound loops that must never call cudaMalloc (it can synchronise the
// whole device and take unbounded time).  fa_backward_noalloc serves them by
// taking its scratch from a fixed array built into this library.
//
// The array lives in device memory of every GPU that loads the library, for
// the life of the process.  All calls on a GPU share it and it keeps the
// previous call's contents.  The backward keeps only two fp32 row vectors
// there (D and the base-2 LSE), and its dQ kernel rewrites both on every
// call before the dK/dV kernel reads them, so nothing carries over from one
// call to the next; but two calls whose kernels overlap on the GPU (for
// example on two streams) race on the array.
namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

std::atomic<void*> g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device (a supported
// device: the caller has checked it).  In host code the array's name is only
// a host-side stand-in, so the address is looked up once per device (with
// that device current) and published with a release store.
fa_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  void* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    p = g_noalloc_ptr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess) return cuda_fail(e);
      g_noalloc_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return FA_OK;
}

}  // namespace

extern "C" fa_status fa_backward_noalloc(const void* q, const void* k, const void* v,
                                         const void* o, const void* dO, const float* lse,
                                         void* dq, void* dk, void* dv, int B, int H, int N,
                                         int d, float scale, int causal, void* stream) {
  // Shape first (the size formula assumes checked sizes), then the size
  // limit (host arithmetic only), then the device: the array's address is
  // only looked up on a device the library's kernels run on.
  fa_status st = check_common(B, H, N, d, scale, FA_BF16);
  if (st != FA_OK) return st;
  if (ws_layout(B, H, N, d).total > static_cast<size_t>(FA_NOALLOC_SCRATCH_BYTES))
    return FA_ERR_WORKSPACE;  // the problem needs more scratch than the array holds
  fa::Launch L;
  st = device_context(stream, &L);
  if (st != FA_OK) return st;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != FA_OK) return st;
  return fa_backward_ex(q, k, v, o, dO, lse, dq, dk, dv, B, H, N, d, scale, causal, scratch,
                        static_cast<size_t>(FA_NOALLOC_SCRATCH_BYTES), FA_BF16, stream);
}

// ---------------------------------------------------------------------------
// FP8 (E4M3) forward and the per-tensor E4M3 quantiser.
namespace {

// [BH, N, d] E4M3 (one byte per element) viewed as 3-D {d, N, BH}; box
// {128, 128, 1}, a whole 128-byte swizzle row per query or key; columns past
// d and rows past N read as zero.
fa_status make_map_e4m3(CUtensorMap* m, const void* base, int BH, int N, int d) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d),
                           static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d)};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_cuda_error = static_cast<int>(r);
    return FA_ERR_CUDA;
  }
  return FA_OK;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" {

fa_status fa_forward_fp8(const void* q, const void* k, const void* v, const float* q_descale,
                         const float* k_descale, const float* v_descale, void* o, float* lse,
                         int B, int H, int N, int d, float scale, int causal, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  fa_status st = check_common(B, H, N, d, scale, FA_BF16);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_MISALIGNED;
  if ((q_descale && !aligned4(q_descale)) || (k_descale && !aligned4(k_descale)) ||
      (v_descale && !aligned4(v_descale)))
    return FA_ERR_MISALIGNED;
  fa::Launch L;
  st = device_context(stream, &L);
  if (st != FA_OK) return st;
  const int BH = B * H;
  st = get_encoder();
  if (st != FA_OK) return st;
  CUtensorMap tq, tk, tv;
  if ((st = make_map_e4m3(&tq, q, BH, N, d)) != FA_OK) return st;
  if ((st = make_map_e4m3(&tk, k, BH, N, d)) != FA_OK) return st;
  if ((st = make_map_e4m3(&tv, v, BH, N, d)) != FA_OK) return st;
  cudaError_t e = fa::launch_fwd_fp8_sm100(tq, tk, tv, q_descale, k_descale, v_descale, o, lse,
                                           BH, N, d, scale, causal ? 1 : 0, L);
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

fa_status fa_quantize_fp8(const void* x, fa_dtype dtype, size_t n, void* codes, float* descale,
                          void* stream) {
  if (!x || !codes || !descale || n == 0) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP32) return FA_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(codes) || !aligned4(descale)) return FA_ERR_MISALIGNED;
  fa::Launch L;
  fa_status st = device_context(stream, &L);
  if (st != FA_OK) return st;
  cudaError_t e = cudaMemsetAsync(descale, 0, sizeof(float), L.stream);
  if (e != cudaSuccess) return cuda_fail(e);
  e = fa::launch_quantize_e4m3(x, dtype == FA_BF16 ? 1 : 0, n, static_cast<uint8_t*>(codes),
                               descale, L);
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

}  // extern "C"
