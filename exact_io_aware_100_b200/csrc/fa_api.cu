// Host side of libfa.so: argument validation, TMA descriptors, launches.
// The C ABI is declared (and documented) in include/fa.h.
#include "fa.h"

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "bwd_kernel.cuh"
#include "decode_kernel.cuh"
#include "fwd_kernel.cuh"

namespace fa {

constexpr int kMaxDevices = 64;
__device__ uint32_t g_status;   // device status word (bits of DEV_*), one per device

namespace {

constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s per bounded wait

struct DevState {
  bool ready = false;
  uint32_t* status = nullptr;
  int sms = 0;
  bool fwd_attr64 = false, fwd_attr128 = false, bwd_attr64 = false, bwd_attr128 = false, dec_attr = false;
};
DevState g_dev[kMaxDevices];
std::mutex g_mu;

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

fa_status device_state(DevState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DevState& s = g_dev[dev];
  if (!s.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return FA_ERR_CUDA;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
      return FA_ERR_CUDA;
    s.status = static_cast<uint32_t*>(p);
    s.sms = sms;
    s.ready = true;
  }
  *out = &s;
  return FA_OK;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

fa_status check_sizes(int B, int H, int N, int d, float scale) {
  if (B < 1 || H < 1 || N < 1 || N > (1 << 24) || !std::isfinite(scale)) return FA_ERR_INVALID;
  const long long numel = 1LL * B * H * N * d;
  if (numel >= (1LL << 31)) return FA_ERR_INVALID;
  return FA_OK;
}

// 3-D bf16 tensor map over [BH][N][d]: box {64 columns, box_rows rows, 1 head},
// 128-byte swizzle (the layout the UMMA descriptors in the kernels expect).
bool make_map(CUtensorMap* m, const void* base, int d, int N, int BH, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

__global__ void cast_f32_bf16_kernel(const float4* __restrict__ src, uint2* __restrict__ dst, size_t n4) {
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 v = src[i];
    uint2 w;
    w.x = pack_bf16x2(v.x, v.y);
    w.y = pack_bf16x2(v.z, v.w);
    dst[i] = w;
  }
}

__global__ void wait_probe_kernel(uint32_t* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0u;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl ctl{&abort_flag, status, limit_ns};
    (void)mbar_wait(smem_u32(&bar), 0, ctl);   // nothing ever arrives: gives up after limit_ns
  }
  __syncthreads();
}

// The register splits inside the kernels (setmaxnreg) are computed for the
// register count each kernel is launched with; a build that compiled to a
// different count would make a setmaxnreg.inc wait forever, so such a kernel
// is never launched.
bool launch_regs_are(const void* fn, int regs) {
  cudaFuncAttributes fa_attr;
  return cudaFuncGetAttributes(&fa_attr, fn) == cudaSuccess && fa_attr.numRegs == regs;
}

template <int D>
fa_status launch_fwd(DevState* ds, const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int H_kv, int N, float scale, int causal, int o_f32, cudaStream_t stream) {
  const int BH = B * H;
  using C = FwdCfg<D>;
  bool& attr = (D == 64) ? ds->fwd_attr64 : ds->fwd_attr128;
  if (!attr) {
    if (!launch_regs_are(reinterpret_cast<const void*>(fa_fwd_kernel<D>), C::LAUNCH_REGS)) return FA_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(fa_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
        cudaSuccess)
      return FA_ERR_CUDA;
    attr = true;
  }
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, D, N, BH, 128) || !make_map(&tk, k, D, N, B * H_kv, 128) ||
      !make_map(&tv, v, D, N, B * H_kv, 128))
    return FA_ERR_CUDA;
  FwdArgs a;
  a.o = o;
  a.lse = lse;
  a.status = ds->status;
  a.N = N;
  a.bh = BH;
  a.heads = H;
  a.group = H / H_kv;
  a.n_qt = (N + 255) / 256;
  a.n_kv_all = (N + 127) / 128;
  a.num_tiles = BH * a.n_qt;
  a.causal = causal ? 1 : 0;
  a.o_f32 = o_f32;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.wait_limit_ns = kWaitLimitNs;
  const int grid = a.num_tiles < ds->sms ? a.num_tiles : ds->sms;
  fa_fwd_kernel<D><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, a);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv, int N,
                   int d, float scale, int causal, fa_dtype dtype, void* ws, size_t ws_bytes, cudaStream_t stream) {
  fa_status st = check_sizes(B, H, N, d, scale);
  if (st != FA_OK) return st;
  if (H_kv < 1 || H % H_kv != 0) return FA_ERR_INVALID;
  if (H_kv != H && dtype != FA_BF16) return FA_ERR_UNSUPPORTED;   // grouped heads: bf16 inputs only
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (dtype != FA_BF16 && dtype != FA_F32) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_ALIGN;
  const size_t need = fa_fwd_workspace_size(B, H, N, d, dtype);
  if (need > 0 && (ws == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)))
    return FA_ERR_WORKSPACE;
  DevState* ds = nullptr;
  if ((st = device_state(&ds)) != FA_OK) return st;
  const int BH = B * H;
  const void *qq = q, *kk = k, *vv = v;
  if (dtype == FA_F32) {
    const size_t n = static_cast<size_t>(BH) * N * d;
    const size_t part = round256(n * 2);
    uint8_t* w = static_cast<uint8_t*>(ws);
    const void* src[3] = {q, k, v};
    for (int i = 0; i < 3; ++i) {
      const size_t n4 = n / 4;
      const int blocks = static_cast<int>((n4 + 255) / 256 < 4096 ? (n4 + 255) / 256 : 4096);
      cast_f32_bf16_kernel<<<blocks, 256, 0, stream>>>(static_cast<const float4*>(src[i]),
                                                        reinterpret_cast<uint2*>(w + i * part), n4);
    }
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    qq = w;
    kk = w + part;
    vv = w + 2 * part;
  }
  const int of32 = dtype == FA_F32 ? 1 : 0;
  return d == 64 ? launch_fwd<64>(ds, qq, kk, vv, o, lse, B, H, H_kv, N, scale, causal, of32, stream)
                 : launch_fwd<128>(ds, qq, kk, vv, o, lse, B, H, H_kv, N, scale, causal, of32, stream);
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" {

size_t fa_fwd_workspace_size(int B, int H, int N, int d, fa_dtype dtype) {
  if (dtype != FA_F32 || B < 1 || H < 1 || N < 1 || d < 1) return 0;
  return 3 * round256(static_cast<size_t>(B) * H * N * d * 2);
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 float scale, int causal, fa_stream_t stream) {
  return fwd_impl(q, k, v, o, lse, B, H, H, N, d, scale, causal, FA_BF16, nullptr, 0,
                  static_cast<cudaStream_t>(stream));
}

fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv,
                     int N, int d, float scale, int causal, fa_stream_t stream) {
  return fwd_impl(q, k, v, o, lse, B, H, H_kv, N, d, scale, causal, FA_BF16, nullptr, 0,
                  static_cast<cudaStream_t>(stream));
}

fa_status fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                    float scale, int causal, fa_dtype dtype, void* workspace, size_t workspace_bytes,
                    fa_stream_t stream) {
  return fwd_impl(q, k, v, o, lse, B, H, H, N, d, scale, causal, dtype, workspace, workspace_bytes,
                  static_cast<cudaStream_t>(stream));
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || d < 1) return 0;
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t np = (static_cast<size_t>(N) + 127) / 128 * 128;
  return round256(bh * N * d * 4) + 2 * round256(bh * np * 4);
}

}  // extern "C"

namespace fa {
namespace {

enum BwdPhase : int { PH_PREPARE = 1, PH_MAIN = 2, PH_FINISH = 4, PH_ALL = 7 };

// First use of the backward main kernel for head dim D on a device.
template <int D>
fa_status prepare_bwd_kernel() {
  using C = BwdCfg<D>;
  if (!launch_regs_are(reinterpret_cast<const void*>(fa_bwd_kernel<D>), C::LAUNCH_REGS)) return FA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(fa_bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  return FA_OK;
}

// Validates, fills the kernel arguments, and launches the requested phases.
fa_status bwd_impl(int phases, const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dout, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N, int d,
                   float scale, int causal, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  fa_status st = check_sizes(B, H, N, d, scale);
  if (st != FA_OK) return st;
  if (H_kv < 1 || H % H_kv != 0) return FA_ERR_INVALID;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if ((phases & PH_PREPARE) && (!aligned16(o) || !aligned16(lse) || !aligned16(dout))) return FA_ERR_ALIGN;
  if ((phases & PH_MAIN) && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) ||
                             !aligned16(dk) || !aligned16(dv)))
    return FA_ERR_ALIGN;
  if ((phases & PH_FINISH) && !aligned16(dq)) return FA_ERR_ALIGN;
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return FA_ERR_WORKSPACE;
  DevState* ds = nullptr;
  if ((st = device_state(&ds)) != FA_OK) return st;
  if ((phases & PH_MAIN) && !(d == 64 ? ds->bwd_attr64 : ds->bwd_attr128)) {
    st = d == 64 ? prepare_bwd_kernel<64>() : prepare_bwd_kernel<128>();
    if (st != FA_OK) return st;
    (d == 64 ? ds->bwd_attr64 : ds->bwd_attr128) = true;
  }
  const int BH = B * H;
  BwdArgs a;
  const size_t np = (static_cast<size_t>(N) + 127) / 128 * 128;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  a.dq_acc = reinterpret_cast<float*>(w);
  a.lse2 = reinterpret_cast<float*>(w + round256(static_cast<size_t>(BH) * N * d * 4));
  a.dvec = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.lse2) + round256(BH * np * 4));
  a.o = static_cast<const __nv_bfloat16*>(o);
  a.dout = static_cast<const __nv_bfloat16*>(dout);
  a.lse = lse;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.status = ds->status;
  a.N = N;
  a.Np = static_cast<int>(np);
  a.bh = BH;
  a.bh_kv = B * H_kv;
  a.heads = H;
  a.group = H / H_kv;
  a.n_kb = (N + 127) / 128;
  a.n_qb = (N + 127) / 128;
  // enough key/value heads per scheduling group to fill the GPU about twice over with key blocks
  const int want = (2 * ds->sms + a.n_kb - 1) / a.n_kb;
  a.heads_per_group = want < 1 ? 1 : (want > a.bh_kv ? a.bh_kv : want);
  a.causal = causal ? 1 : 0;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.wait_limit_ns = kWaitLimitNs;
  if (phases & PH_PREPARE) {
    if (d == 64)
      fa_bwd_pre_kernel<64><<<ds->sms * 8, 256, 0, stream>>>(a);
    else
      fa_bwd_pre_kernel<128><<<ds->sms * 8, 256, 0, stream>>>(a);
  }
  if (phases & PH_MAIN) {
    CUtensorMap tq, tk, tv, tdo;
    if (!make_map(&tq, q, d, N, BH, 128) || !make_map(&tk, k, d, N, a.bh_kv, 128) ||
        !make_map(&tv, v, d, N, a.bh_kv, 128) || !make_map(&tdo, dout, d, N, BH, 128))
      return FA_ERR_CUDA;
    if (d == 64)
      fa_bwd_kernel<64><<<a.n_kb * a.bh_kv, BwdCfg<64>::THREADS, BwdCfg<64>::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, a);
    else
      fa_bwd_kernel<128><<<a.n_kb * a.bh_kv, BwdCfg<128>::THREADS, BwdCfg<128>::SMEM_BYTES, stream>>>(tq, tk, tv, tdo,
                                                                                                       a);
  }
  if (phases & PH_FINISH) {
    if (d == 64)
      fa_bwd_dq_kernel<64><<<ds->sms * 8, 256, 0, stream>>>(a);
    else
      fa_bwd_dq_kernel<128><<<ds->sms * 8, 256, 0, stream>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace
}  // namespace fa

extern "C" {

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                 void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                 void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  return bwd_impl(PH_ALL, q, k, v, o, lse, dout, dq, dk, dv, B, H, H, N, d, scale, causal, workspace,
                  workspace_bytes, static_cast<cudaStream_t>(stream));
}

fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N, int d,
                     float scale, int causal, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  return bwd_impl(PH_ALL, q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, d, scale, causal, workspace,
                  workspace_bytes, static_cast<cudaStream_t>(stream));
}

fa_status fa_bwd_prepare(const void* o, const float* lse, const void* dout, int B, int H, int N, int d,
                         void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  return bwd_impl(PH_PREPARE, nullptr, nullptr, nullptr, o, lse, dout, nullptr, nullptr, nullptr, B, H, H, N, d,
                  1.0f, 0, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

fa_status fa_bwd_main(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv, int B,
                      int H, int N, int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                      fa_stream_t stream) {
  return bwd_impl(PH_MAIN, q, k, v, nullptr, nullptr, dout, nullptr, dk, dv, B, H, H, N, d, scale, causal,
                  workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

fa_status fa_bwd_finish(void* dq, int B, int H, int N, int d, float scale, void* workspace,
                        size_t workspace_bytes, fa_stream_t stream) {
  return bwd_impl(PH_FINISH, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, dq, nullptr, nullptr, B, H,
                  H, N, d, scale, 0, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

// ---- backward with built-in scratch (no allocation) ----
// One fixed-size device array per device that loads the library; every
// fa_bwd_noalloc call on that device uses it as the fa_bwd workspace.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_ptr[fa::kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch on the current device (looked up once per
// device; the host-side symbol itself is not a device address).
fa_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= fa::kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return FA_OK;
}
}  // namespace

fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
                         int causal, fa_stream_t stream) {
  fa_status st = check_sizes(B, H, N, d, scale);
  if (st != FA_OK) return st;
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (need > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_WORKSPACE;   // beyond the built-in scratch
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != FA_OK) return st;
  return fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, scratch,
                FA_NOALLOC_SCRATCH_BYTES, stream);
}

fa_status fa_get_device_status(fa_stream_t stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  uint32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return FA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
  if (v & DEV_TIMEOUT) return FA_ERR_TIMEOUT;
  return (v & DEV_SMEM) ? FA_ERR_CUDA : FA_OK;
}

fa_status fa_selftest_wait_timeout(uint64_t timeout_ns, fa_stream_t stream) {
  DevState* ds = nullptr;
  fa_status st = device_state(&ds);
  if (st != FA_OK) return st;
  uint64_t t = timeout_ns < 1000000ull ? 1000000ull : timeout_ns;
  if (t > kWaitLimitNs) t = kWaitLimitNs;
  wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ds->status, t);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_decode_workspace_size(int B, int H, int H_kv, int Lq, int Nk, int d) {
  if (B < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || Lq < 1 || Nk < Lq || d < 1) return 0;
  int split_keys = 0;
  const size_t splits = static_cast<size_t>(decode_splits(B * H_kv, Nk, &split_keys));
  const size_t rows = static_cast<size_t>(B) * H * Lq;
  return round256(splits * rows * d * 4) + round256(splits * rows * 4);
}

fa_status fa_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv,
                    int Lq, int Nk, int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                    fa_stream_t stream) {
  fa_status st = check_sizes(B, H_kv, Nk, d, scale);
  if (st != FA_OK) return st;
  if (Lq < 1 || Lq > Nk || H < 1 || H_kv > H || H % H_kv != 0 || 1LL * B * H * Lq * d >= (1LL << 31) ||
      B * H_kv > 65535)
    return FA_ERR_INVALID;
  if (d != DecCfg::D || (H / H_kv) * Lq > DecCfg::R_MAX) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_ALIGN;
  const size_t need = fa_decode_workspace_size(B, H, H_kv, Lq, Nk, d);
  if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return FA_ERR_WORKSPACE;
  DevState* ds = nullptr;
  if ((st = device_state(&ds)) != FA_OK) return st;
  if (!ds->dec_attr) {
    if (cudaFuncSetAttribute(fa_decode_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, DecCfg::SMEM_BYTES) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fa_decode_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, DecCfg::SMEM_BYTES) !=
            cudaSuccess ||
        cudaFuncSetAttribute(fa_decode_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, DecCfg::SMEM_BYTES) !=
            cudaSuccess)
      return FA_ERR_CUDA;
    ds->dec_attr = true;
  }
  CUtensorMap tk, tv;
  if (!make_map(&tk, k, d, Nk, B * H_kv, DecCfg::KT) || !make_map(&tv, v, d, Nk, B * H_kv, DecCfg::KT))
    return FA_ERR_CUDA;
  DecArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.status = ds->status;
  a.Lq = Lq;
  a.Nk = Nk;
  a.heads = H;
  a.group = H / H_kv;
  a.bh = B * H;
  a.bh_kv = B * H_kv;
  a.n_splits = decode_splits(a.bh_kv, Nk, &a.split_keys);
  a.causal = causal ? 1 : 0;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.wait_limit_ns = kWaitLimitNs;
  const size_t rows = static_cast<size_t>(a.bh) * Lq;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  a.part_o = reinterpret_cast<float*>(w);
  a.part_lse = reinterpret_cast<float*>(w + round256(static_cast<size_t>(a.n_splits) * rows * d * 4));
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const dim3 grid(a.n_splits, a.bh_kv);
  const int rows_per_set = a.group * Lq;
  if (rows_per_set <= 4)
    fa_decode_kernel<4><<<grid, DecCfg::THREADS, DecCfg::SMEM_BYTES, s>>>(tk, tv, a);
  else if (rows_per_set <= 8)
    fa_decode_kernel<8><<<grid, DecCfg::THREADS, DecCfg::SMEM_BYTES, s>>>(tk, tv, a);
  else
    fa_decode_kernel<16><<<grid, DecCfg::THREADS, DecCfg::SMEM_BYTES, s>>>(tk, tv, a);
  const size_t warps = rows, per_block = 8;
  size_t blocks = (warps + per_block - 1) / per_block;
  if (blocks > static_cast<size_t>(ds->sms) * 16) blocks = static_cast<size_t>(ds->sms) * 16;
  fa_decode_merge_kernel<<<static_cast<unsigned>(blocks), 32 * per_block, 0, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID: return "FA_ERR_INVALID";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_ALIGN: return "FA_ERR_ALIGN";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
  }
  return "FA_ERR_UNKNOWN";
}

const char* fa_version(void) { return "0.1.0"; }

}  // extern "C"
