// Host side of libfa.so: argument validation, TMA descriptors, launches.
// The C ABI is declared (and documented) in include/fa.h.
#include "fa.h"

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <type_traits>

#include "bwd256_kernel.cuh"
#include "bwd_kernel.cuh"
#include "decode_kernel.cuh"
#include "decode_warp_kernel.cuh"
#include "fwd256_kernel.cuh"
#include "fwd64_kernel.cuh"
#include "fwd_kernel.cuh"

namespace fa {

constexpr int kMaxDevices = 64;
__device__ uint32_t g_status;   // device status word (bits of DEV_*), one per device

namespace {

constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s per bounded wait

struct DevState {
  bool ready = false;
  unsigned long long ctx_id = 0;                   // context the state below was set up in
  uint32_t* status = nullptr;
  int sms = 0;
  bool fwd_attr[2][2] = {}, bwd_attr[2][2] = {};   // [d == 128][packed]: attributes set, registers checked
  bool bwd256_attr[2] = {};                        // [packed]
  bool fwd256_attr[2] = {};                        // [packed]
  bool dec_attr = false, decw_attr = false;
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

}  // namespace

// Unique id of the CUDA context current on this thread, 0 if there is none yet.
// Device addresses of the library's __device__ arrays and the kernel attributes
// belong to a context: after a device reset (a new primary context) they are
// looked up and set again.
unsigned long long current_ctx_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

namespace {

fa_status device_state(DevState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DevState& s = g_dev[dev];
  if (!s.ready || s.ctx_id != current_ctx_id()) {
    s = DevState();
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return FA_ERR_CUDA;   // makes the context current
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
      return FA_ERR_CUDA;
    s.status = static_cast<uint32_t*>(p);
    s.sms = sms;
    s.ctx_id = current_ctx_id();
    s.ready = true;
  }
  *out = &s;
  return FA_OK;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// The score scale must be finite and positive: the kernels take the row
// maximum of the unscaled scores as the softmax reference.
bool scale_ok(float scale) { return std::isfinite(scale) && scale > 0.0f; }

fa_status check_sizes(int B, int H, int N, int d, float scale) {
  if (B < 1 || H < 1 || N < 1 || N > (1 << 24) || !scale_ok(scale)) return FA_ERR_INVALID;
  const long long numel = 1LL * B * H * N * d;
  if (numel >= (1LL << 31)) return FA_ERR_INVALID;
  return FA_OK;
}

// 4-D bf16 tensor map over [batch][head][row][d] with element strides st:
// box {64 columns, box_rows rows, 1 head, 1 batch entry}, 128-byte swizzle
// (the layout the UMMA descriptors in the kernels expect).  Extents of 1 get a
// harmless dense stride (the copy never steps along them); an extent of 0
// rows is mapped as 1 row that no copy reads.
bool make_map4(CUtensorMap* m, const void* base, int d, int rows, int heads, int batches, const fa_strides& st,
               int box_rows = 128) {
  auto fn = encode_fn();
  if (!fn) return false;
  if (rows < 1) rows = 1;
  const cuuint64_t dense = static_cast<cuuint64_t>(d) * 2;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(batches)};
  cuuint64_t strides[3] = {rows > 1 ? static_cast<cuuint64_t>(st.row) * 2 : dense,
                           heads > 1 ? static_cast<cuuint64_t>(st.head) * 2 : dense,
                           batches > 1 ? static_cast<cuuint64_t>(st.batch) * 2 : dense};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D map of the fp32 dQ accumulator at head dim 256, [rows][256], for the
// backward's tensor bulk reductions: box of 128 columns (one CTA's half of d) by
// `box_rows` rows, no swizzle.
bool make_map_dq256(CUtensorMap* m, float* acc, long long rows, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {256, static_cast<cuuint64_t>(rows < 1 ? 1 : rows)};
  cuuint64_t strides[1] = {256 * 4};
  cuuint32_t box[2] = {128, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, acc, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

fa_strides dense_strides(int H, int N, int d) {
  fa_strides st;
  st.row = d;
  st.head = static_cast<int64_t>(N) * d;
  st.batch = static_cast<int64_t>(H) * N * d;
  return st;
}

// The layout of dense [B, H, N, d] tensors (H_kv heads for k, v, dk, dv).
fa_layout dense_layout(int B, int H, int H_kv, int N, int d) {
  fa_layout L = {};
  L.B = B;
  L.H = H;
  L.H_kv = H_kv;
  L.d = d;
  L.Nq = L.Nk = N;
  L.cu_seqlens_q = L.cu_seqlens_k = nullptr;
  L.total_q = L.total_k = 0;
  L.q = L.o = L.dout = L.dq = dense_strides(H, N, d);
  L.k = L.v = L.dk = L.dv = dense_strides(H_kv, N, d);
  return L;
}

bool packed(const fa_layout& L) { return L.cu_seqlens_q != nullptr; }
int q_rows(const fa_layout& L) { return packed(L) ? L.total_q : L.Nq; }   // row extent of q-like tensors
int k_rows(const fa_layout& L) { return packed(L) ? L.total_k : L.Nk; }
int batches(const fa_layout& L) { return packed(L) ? 1 : L.B; }

// Strides usable by TMA and by 16-byte row stores: positive multiples of 8
// elements (16 bytes of bf16) below 2^38 (a tensor map stride is under 2^40 B).
bool strides_ok(const fa_strides& st, int rows, int heads, int batches) {
  auto ok = [](int64_t x, int extent) { return extent <= 1 || (x > 0 && x % 8 == 0 && x < (int64_t(1) << 38)); };
  return ok(st.row, rows) && ok(st.head, heads) && ok(st.batch, batches);
}

// Sizes and strides of a layout (the pointers are checked by the caller).
fa_status check_layout(const fa_layout& L, bool bwd) {
  if (L.B < 1 || L.H < 1 || L.H_kv < 1 || L.H % L.H_kv != 0) return FA_ERR_INVALID;
  if (L.Nq < 0 || L.Nk < 0 || L.Nq > (1 << 24) || L.Nk > (1 << 24)) return FA_ERR_INVALID;
  if ((L.cu_seqlens_q == nullptr) != (L.cu_seqlens_k == nullptr)) return FA_ERR_INVALID;
  if (packed(L)) {
    if (L.total_q < 0 || L.total_k < 0 || L.B > (1 << 24)) return FA_ERR_INVALID;
    if (reinterpret_cast<uintptr_t>(L.cu_seqlens_q) % 4 || reinterpret_cast<uintptr_t>(L.cu_seqlens_k) % 4)
      return FA_ERR_ALIGN;
  }
  if (L.d != 64 && L.d != 128 && L.d != 256) return FA_ERR_UNSUPPORTED;
  // every row index the kernels form stays below 2^31
  const long long qr = static_cast<long long>(batches(L)) * L.H * (packed(L) ? L.total_q : L.Nq);
  const long long pr = static_cast<long long>(L.B) * L.H * ((static_cast<long long>(L.Nq) + 127) / 128 * 128);
  if (qr >= (1LL << 31) || pr >= (1LL << 31)) return FA_ERR_INVALID;
  const int bq = batches(L), nq = q_rows(L), nk = k_rows(L);
  if (!strides_ok(L.q, nq, L.H, bq) || !strides_ok(L.o, nq, L.H, bq) || !strides_ok(L.k, nk, L.H_kv, bq) ||
      !strides_ok(L.v, nk, L.H_kv, bq))
    return FA_ERR_ALIGN;
  if (bwd && (!strides_ok(L.dout, nq, L.H, bq) || !strides_ok(L.dq, nq, L.H, bq) ||
              !strides_ok(L.dk, nk, L.H_kv, bq) || !strides_ok(L.dv, nk, L.H_kv, bq)))
    return FA_ERR_ALIGN;
  return FA_OK;
}

SeqLayout seq_layout(const fa_layout& L) {
  SeqLayout s;
  s.cu_q = L.cu_seqlens_q;
  s.cu_k = L.cu_seqlens_k;
  s.B = L.B;
  s.H = L.H;
  s.H_kv = L.H_kv;
  s.Nq = L.Nq;
  s.Nk = L.Nk;
  s.total_q = L.total_q;
  s.total_k = L.total_k;
  return s;
}

Strides kstrides(const fa_strides& st) { return Strides{st.batch, st.head, st.row}; }

// Causal forward tile order: query heads taken in groups whose keys and values
// (at most Nk rows each, bf16) fit in about 48 MB of L2 together, so the CTAs
// working on a group's tiles share them there; whole key/value-head sets.
int fwd_heads_per_group(const fa_layout& L) {
  const double kv_bytes = 4.0 * (L.Nk > 0 ? L.Nk : 1) * L.d;   // K and V of one key/value head
  long long kv_heads = static_cast<long long>(48.0 * (1 << 20) / kv_bytes);
  if (kv_heads < 1) kv_heads = 1;
  const long long hg = kv_heads * (L.H / L.H_kv);
  const long long bh_all = static_cast<long long>(L.B) * L.H;
  return static_cast<int>(hg < bh_all ? hg : bh_all);
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

// q, k and v (blockIdx.y) rounded to bf16 in one launch: each is n4 float4 groups.
struct CastArgs {
  const float4* src[3];
  uint2* dst[3];
};
__global__ void cast_f32_bf16_kernel(const CastArgs a, size_t n4) {
  const float4* __restrict__ src = a.src[blockIdx.y];
  uint2* __restrict__ dst = a.dst[blockIdx.y];
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

// The forward kernel a head dim uses: at d = 64 the one with separate P buffers
// (next scores computed during the softmax), at d = 128 the ping-pong kernel.
template <int D>
struct FwdPlan;
template <>
struct FwdPlan<64> {
  using C = FwdSpCfg<64, 128>;
  template <bool PACKED>
  static constexpr auto kernel() { return fa_fwd_sp_kernel<64, 128, PACKED>; }
};
template <>
struct FwdPlan<128> {
  using C = FwdCfg<128>;
  template <bool PACKED>
  static constexpr auto kernel() { return fa_fwd_kernel<128, PACKED>; }
};

template <int D>
fa_status launch_fwd(DevState* ds, const void* q, const void* k, const void* v, void* o, float* lse,
                     const fa_layout& L, float scale, int causal, int o_f32, cudaStream_t stream) {
  using C = typename FwdPlan<D>::C;
  const bool pk = packed(L);
  auto kern = pk ? FwdPlan<D>::template kernel<true>() : FwdPlan<D>::template kernel<false>();
  bool& attr = ds->fwd_attr[D == 128][pk];
  if (!attr) {
    if (!launch_regs_are(reinterpret_cast<const void*>(kern), C::LAUNCH_REGS)) return FA_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
      return FA_ERR_CUDA;
    attr = true;
  }
  if (L.Nq == 0 || (packed(L) && L.total_q == 0)) return FA_OK;   // no query row: nothing to write
  CUtensorMap tq, tk, tv;
  const int bq = batches(L);
  if (!make_map4(&tq, q, D, q_rows(L), L.H, bq, L.q) || !make_map4(&tk, k, D, k_rows(L), L.H_kv, bq, L.k, C::BN) ||
      !make_map4(&tv, v, D, k_rows(L), L.H_kv, bq, L.v, C::BN))
    return FA_ERR_CUDA;
  FwdArgs a;
  a.o = o;
  a.lse = lse;
  a.status = ds->status;
  a.L = seq_layout(L);
  a.so = kstrides(L.o);
  a.group = L.H / L.H_kv;
  a.n_qt = (L.Nq + 255) / 256;
  a.num_tiles = L.B * L.H * a.n_qt;
  a.heads_per_group = fwd_heads_per_group(L);
  a.causal = causal ? 1 : 0;
  a.o_f32 = o_f32;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.wait_limit_ns = kWaitLimitNs;
  const int grid = a.num_tiles < ds->sms ? a.num_tiles : ds->sms;
  kern<<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, a);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Head dim 256 (forward, bf16): one 128-row query tile per CTA, 64-key blocks.
template <bool PACKED>
fa_status launch_fwd256_t(DevState* ds, const void* q, const void* k, const void* v, void* o, float* lse,
                          const fa_layout& L, float scale, int causal, cudaStream_t stream) {
  using C = Fwd256Cfg;
  if (!ds->fwd256_attr[PACKED]) {
    if (cudaFuncSetAttribute(fa_fwd256_kernel<PACKED>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
        cudaSuccess)
      return FA_ERR_CUDA;
    ds->fwd256_attr[PACKED] = true;
  }
  CUtensorMap tq, tk, tv;
  const int bq = batches(L);
  if (!make_map4(&tq, q, 256, q_rows(L), L.H, bq, L.q, 128) || !make_map4(&tk, k, 256, k_rows(L), L.H_kv, bq, L.k, 64) ||
      !make_map4(&tv, v, 256, k_rows(L), L.H_kv, bq, L.v, 64))
    return FA_ERR_CUDA;
  FwdArgs a;
  a.o = o;
  a.lse = lse;
  a.status = ds->status;
  a.L = seq_layout(L);
  a.so = kstrides(L.o);
  a.group = L.H / L.H_kv;
  a.n_qt = (L.Nq + 127) / 128;
  a.num_tiles = L.B * L.H * a.n_qt;
  a.heads_per_group = fwd_heads_per_group(L);
  a.causal = causal ? 1 : 0;
  a.o_f32 = 0;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.wait_limit_ns = kWaitLimitNs;
  const int grid = a.num_tiles < ds->sms ? a.num_tiles : ds->sms;
  fa_fwd256_kernel<PACKED><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, a);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status launch_fwd256(DevState* ds, const void* q, const void* k, const void* v, void* o, float* lse,
                        const fa_layout& L, float scale, int causal, cudaStream_t stream) {
  if (L.Nq == 0 || (packed(L) && L.total_q == 0)) return FA_OK;   // no query row: nothing to write
  if (static_cast<long long>(L.B) * L.H * ((L.Nq + 127) / 128) >= (1LL << 31)) return FA_ERR_INVALID;
  return packed(L) ? launch_fwd256_t<true>(ds, q, k, v, o, lse, L, scale, causal, stream)
                   : launch_fwd256_t<false>(ds, q, k, v, o, lse, L, scale, causal, stream);
}

fa_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv, int N,
                   int d, float scale, int causal, fa_dtype dtype, void* ws, size_t ws_bytes, cudaStream_t stream) {
  fa_status st = check_sizes(B, H, N, d, scale);
  if (st != FA_OK) return st;
  if (H_kv < 1 || H % H_kv != 0) return FA_ERR_INVALID;
  if (H_kv != H && dtype != FA_BF16) return FA_ERR_UNSUPPORTED;   // grouped heads: bf16 inputs only
  if (d != 64 && d != 128 && !(d == 256 && dtype == FA_BF16)) return FA_ERR_UNSUPPORTED;
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
    CastArgs ca;
    for (int i = 0; i < 3; ++i) {
      ca.src[i] = static_cast<const float4*>(src[i]);
      ca.dst[i] = reinterpret_cast<uint2*>(w + i * part);
    }
    const size_t n4 = n / 4;
    const unsigned blocks = static_cast<unsigned>((n4 + 255) / 256 < 4096 ? (n4 + 255) / 256 : 4096);
    cast_f32_bf16_kernel<<<dim3(blocks, 3), 256, 0, stream>>>(ca, n4);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    qq = w;
    kk = w + part;
    vv = w + 2 * part;
  }
  const int of32 = dtype == FA_F32 ? 1 : 0;
  const fa_layout L = dense_layout(B, H, H_kv, N, d);
  if (d == 256) return launch_fwd256(ds, qq, kk, vv, o, lse, L, scale, causal, stream);
  return d == 64 ? launch_fwd<64>(ds, qq, kk, vv, o, lse, L, scale, causal, of32, stream)
                 : launch_fwd<128>(ds, qq, kk, vv, o, lse, L, scale, causal, of32, stream);
}

fa_status fwd_general_impl(const void* q, const void* k, const void* v, void* o, float* lse, const fa_layout* Lp,
                           float scale, int causal, cudaStream_t stream) {
  if (Lp == nullptr) return FA_ERR_INVALID;
  const fa_layout& L = *Lp;
  fa_status st = check_layout(L, false);
  if (st != FA_OK) return st;
  if (!scale_ok(scale)) return FA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_ALIGN;
  DevState* ds = nullptr;
  if ((st = device_state(&ds)) != FA_OK) return st;
  if (L.d == 256) return launch_fwd256(ds, q, k, v, o, lse, L, scale, causal, stream);
  return L.d == 64 ? launch_fwd<64>(ds, q, k, v, o, lse, L, scale, causal, 0, stream)
                   : launch_fwd<128>(ds, q, k, v, o, lse, L, scale, causal, 0, stream);
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

fa_status fa_fwd_general(const void* q, const void* k, const void* v, void* o, float* lse, const fa_layout* layout,
                         float scale, int causal, fa_stream_t stream) {
  return fwd_general_impl(q, k, v, o, lse, layout, scale, causal, static_cast<cudaStream_t>(stream));
}

namespace {
// fp32 dQ accumulator (one row per query row and head), then lse * log2(e) and
// D for rows padded to a multiple of 128 per (sequence, head).
size_t bwd_ws_bytes(const fa_layout& L) {
  const size_t acc_rows = packed(L) ? static_cast<size_t>(L.H) * L.total_q : static_cast<size_t>(L.B) * L.H * L.Nq;
  const size_t np = (static_cast<size_t>(L.Nq) + 127) / 128 * 128;
  return round256(acc_rows * L.d * 4) + 2 * round256(static_cast<size_t>(L.B) * L.H * np * 4);
}
}  // namespace

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || d < 1) return 0;
  return bwd_ws_bytes(dense_layout(B, H, H, N, d));
}

size_t fa_bwd_general_workspace_size(const fa_layout* layout) {
  if (layout == nullptr || check_layout(*layout, true) != FA_OK) return 0;
  return bwd_ws_bytes(*layout);
}

}  // extern "C"

namespace fa {
namespace {

enum BwdPhase : int { PH_PREPARE = 1, PH_MAIN = 2, PH_FINISH = 4, PH_ALL = 7 };

// First use of a backward main kernel on a device.
template <int D, bool PACKED>
fa_status prepare_bwd_kernel() {
  using C = BwdCfg<D>;
  if (!launch_regs_are(reinterpret_cast<const void*>(fa_bwd_kernel<D, PACKED>), C::LAUNCH_REGS))
    return FA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(fa_bwd_kernel<D, PACKED>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  return FA_OK;
}

template <bool PACKED>
fa_status prepare_bwd256_kernel() {
  if (!launch_regs_are(reinterpret_cast<const void*>(fa_bwd256_kernel<PACKED>), Bwd256Cfg::LAUNCH_REGS))
    return FA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(fa_bwd256_kernel<PACKED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Bwd256Cfg::SMEM_BYTES) != cudaSuccess)
    return FA_ERR_CUDA;
  return FA_OK;
}

template <int D>
void launch_bwd_main(bool pk, unsigned grid, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& tdo, const BwdArgs& a, cudaStream_t stream) {
  using C = BwdCfg<D>;
  if (pk)
    fa_bwd_kernel<D, true><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, a);
  else
    fa_bwd_kernel<D, false><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, a);
}

// Validates, fills the kernel arguments, and launches the requested phases.
fa_status bwd_impl(int phases, const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dout, void* dq, void* dk, void* dv, const fa_layout& L, float scale, int causal,
                   void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  fa_status st = check_layout(L, true);
  if (st != FA_OK) return st;
  if (!scale_ok(scale)) return FA_ERR_INVALID;
  const int d = L.d;
  if ((phases & PH_PREPARE) && (!aligned16(o) || !aligned16(lse) || !aligned16(dout))) return FA_ERR_ALIGN;
  if ((phases & PH_MAIN) && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) ||
                             !aligned16(dk) || !aligned16(dv)))
    return FA_ERR_ALIGN;
  if ((phases & PH_FINISH) && !aligned16(dq)) return FA_ERR_ALIGN;
  const size_t need = bwd_ws_bytes(L);
  if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return FA_ERR_WORKSPACE;
  DevState* ds = nullptr;
  if ((st = device_state(&ds)) != FA_OK) return st;
  const bool pk = packed(L);
  if ((phases & PH_MAIN) && d == 256 && !ds->bwd256_attr[pk]) {
    st = pk ? prepare_bwd256_kernel<true>() : prepare_bwd256_kernel<false>();
    if (st != FA_OK) return st;
    ds->bwd256_attr[pk] = true;
  } else if ((phases & PH_MAIN) && d != 256 && !ds->bwd_attr[d == 128][pk]) {
    st = d == 64 ? (pk ? prepare_bwd_kernel<64, true>() : prepare_bwd_kernel<64, false>())
                 : (pk ? prepare_bwd_kernel<128, true>() : prepare_bwd_kernel<128, false>());
    if (st != FA_OK) return st;
    ds->bwd_attr[d == 128][pk] = true;
  }
  BwdArgs a;
  const size_t np = (static_cast<size_t>(L.Nq) + 127) / 128 * 128;
  a.acc_rows = packed(L) ? static_cast<long long>(L.H) * L.total_q : static_cast<long long>(L.B) * L.H * L.Nq;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  a.dq_acc = reinterpret_cast<float*>(w);
  a.lse2 = reinterpret_cast<float*>(w + round256(static_cast<size_t>(a.acc_rows) * d * 4));
  a.dvec = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.lse2) +
                                    round256(static_cast<size_t>(L.B) * L.H * np * 4));
  a.o = static_cast<const __nv_bfloat16*>(o);
  a.dout = static_cast<const __nv_bfloat16*>(dout);
  a.lse = lse;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.status = ds->status;
  a.L = seq_layout(L);
  a.so = kstrides(L.o);
  a.sdo = kstrides(L.dout);
  a.sdq = kstrides(L.dq);
  a.sdk = kstrides(L.dk);
  a.sdv = kstrides(L.dv);
  const fa_strides dd = dense_strides(L.H, L.Nq, d);
  a.dq_dense = !packed(L) && (L.Nq <= 1 || L.dq.row == dd.row) && (L.H <= 1 || L.dq.head == dd.head) &&
               (L.B <= 1 || L.dq.batch == dd.batch);
  a.Np = static_cast<int>(np);
  a.bh_kv = L.B * L.H_kv;
  a.group = L.H / L.H_kv;
  a.n_kb = (L.Nk + 127) / 128;
  // Scheduling groups of key/value heads: enough query heads' key blocks to fill the GPU about
  // four times over, counted in query heads, because a key/value head's items walk every query
  // head of its set; the group's Q, dO and fp32 dQ accumulators (8 bytes per element at d = 128)
  // then stay within L2 (e.g. 9 query heads of 8192 rows: 75 MB).  Measured against one and two
  // fills: equal for multi-head attention, 6.5% faster than two with grouped heads.
  // (at d = 256 two CTAs share each key block, so a fill holds half as many blocks)
  const int nkb = a.n_kb < 1 ? 1 : a.n_kb;
  const int fills = d == 256 ? 2 * ds->sms : 4 * ds->sms;
  const int want = (fills + nkb - 1) / nkb / a.group;
  a.heads_per_group = want < 1 ? 1 : (want > a.bh_kv ? a.bh_kv : want);
  a.causal = causal ? 1 : 0;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.wait_limit_ns = kWaitLimitNs;
  if (phases & PH_PREPARE) {
    if (d == 64)
      fa_bwd_pre_kernel<64><<<ds->sms * 8, 256, 0, stream>>>(a);
    else if (d == 128)
      fa_bwd_pre_kernel<128><<<ds->sms * 8, 256, 0, stream>>>(a);
    else
      fa_bwd_pre_kernel<256><<<ds->sms * 8, 256, 0, stream>>>(a);
  }
  if ((phases & PH_MAIN) && a.n_kb > 0 && !(packed(L) && L.total_k == 0)) {
    CUtensorMap tq, tk, tv, tdo;
    const int bq = batches(L);
    const int qbox = d == 256 ? Bwd256Cfg::BM : 128;   // rows of a query block
    if (!make_map4(&tq, q, d, q_rows(L), L.H, bq, L.q, qbox) || !make_map4(&tk, k, d, k_rows(L), L.H_kv, bq, L.k) ||
        !make_map4(&tv, v, d, k_rows(L), L.H_kv, bq, L.v) ||
        !make_map4(&tdo, dout, d, q_rows(L), L.H, bq, L.dout, qbox))
      return FA_ERR_CUDA;
    const long long grid = static_cast<long long>(a.n_kb) * a.bh_kv * (d == 256 ? 2 : 1);
    if (grid >= (1LL << 31)) return FA_ERR_INVALID;
    if (d == 256) {
      CUtensorMap tdq;
      if (!make_map_dq256(&tdq, a.dq_acc, a.acc_rows, Bwd256Cfg::CHUNK_ROWS)) return FA_ERR_CUDA;
      if (pk)
        fa_bwd256_kernel<true><<<static_cast<unsigned>(grid), Bwd256Cfg::THREADS, Bwd256Cfg::SMEM_BYTES, stream>>>(
            tq, tk, tv, tdo, tdq, a);
      else
        fa_bwd256_kernel<false><<<static_cast<unsigned>(grid), Bwd256Cfg::THREADS, Bwd256Cfg::SMEM_BYTES, stream>>>(
            tq, tk, tv, tdo, tdq, a);
    } else if (d == 64)
      launch_bwd_main<64>(pk, static_cast<unsigned>(grid), tq, tk, tv, tdo, a, stream);
    else
      launch_bwd_main<128>(pk, static_cast<unsigned>(grid), tq, tk, tv, tdo, a, stream);
  }
  if ((phases & PH_FINISH) && a.acc_rows > 0) {
    if (d == 64)
      fa_bwd_dq_kernel<64><<<ds->sms * 8, 256, 0, stream>>>(a);
    else if (d == 128)
      fa_bwd_dq_kernel<128><<<ds->sms * 8, 256, 0, stream>>>(a);
    else
      fa_bwd_dq_kernel<256><<<ds->sms * 8, 256, 0, stream>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace
}  // namespace fa

extern "C" {

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                 void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                 void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  if (check_sizes(B, H, N, d, scale) != FA_OK) return FA_ERR_INVALID;
  return bwd_impl(PH_ALL, q, k, v, o, lse, dout, dq, dk, dv, dense_layout(B, H, H, N, d), scale, causal, workspace,
                  workspace_bytes, static_cast<cudaStream_t>(stream));
}

fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, int B, int H, int H_kv, int N, int d,
                     float scale, int causal, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  if (check_sizes(B, H, N, d, scale) != FA_OK || H_kv < 1) return FA_ERR_INVALID;
  return bwd_impl(PH_ALL, q, k, v, o, lse, dout, dq, dk, dv, dense_layout(B, H, H_kv, N, d), scale, causal,
                  workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

fa_status fa_bwd_general(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv, const fa_layout* layout, float scale,
                         int causal, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  if (layout == nullptr) return FA_ERR_INVALID;
  return bwd_impl(PH_ALL, q, k, v, o, lse, dout, dq, dk, dv, *layout, scale, causal, workspace, workspace_bytes,
                  static_cast<cudaStream_t>(stream));
}

fa_status fa_bwd_prepare(const void* o, const float* lse, const void* dout, int B, int H, int N, int d,
                         void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  if (check_sizes(B, H, N, d, 1.0f) != FA_OK) return FA_ERR_INVALID;
  return bwd_impl(PH_PREPARE, nullptr, nullptr, nullptr, o, lse, dout, nullptr, nullptr, nullptr,
                  dense_layout(B, H, H, N, d), 1.0f, 0, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

fa_status fa_bwd_main(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv, int B,
                      int H, int N, int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                      fa_stream_t stream) {
  if (check_sizes(B, H, N, d, scale) != FA_OK) return FA_ERR_INVALID;
  return bwd_impl(PH_MAIN, q, k, v, nullptr, nullptr, dout, nullptr, dk, dv, dense_layout(B, H, H, N, d), scale,
                  causal, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

fa_status fa_bwd_finish(void* dq, int B, int H, int N, int d, float scale, void* workspace,
                        size_t workspace_bytes, fa_stream_t stream) {
  if (check_sizes(B, H, N, d, scale) != FA_OK) return FA_ERR_INVALID;
  return bwd_impl(PH_FINISH, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, dq, nullptr, nullptr,
                  dense_layout(B, H, H, N, d), scale, 0, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

// ---- backward with built-in scratch (no allocation) ----
// One fixed-size device array per device that loads the library; every
// fa_bwd_noalloc call on that device uses it as the fa_bwd workspace.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_ptr[fa::kMaxDevices] = {};
unsigned long long g_noalloc_ctx[fa::kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch on the current device (the host-side
// symbol itself is not a device address), looked up on the first call in each
// context of the device: once per device unless the device is reset.
fa_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= fa::kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr || g_noalloc_ctx[dev] != fa::current_ctx_id()) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = fa::current_ctx_id();
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
  if (v & DEV_SMEM) return FA_ERR_CUDA;
  return (v & DEV_ARGS) ? FA_ERR_INVALID : FA_OK;
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
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_ALIGN;
  if (d != DecCfg::D || (H / H_kv) * Lq > DecCfg::R_MAX) {
    // outside the split-key decode kernel's shape (d = 128, at most 16 query rows per key/value
    // head): the general forward computes the same result (N_q = Lq queries, bottom-right causal)
    fa_layout L = {};
    L.B = B;
    L.H = H;
    L.H_kv = H_kv;
    L.d = d;
    L.Nq = Lq;
    L.Nk = Nk;
    L.q = L.o = dense_strides(H, Lq, d);
    L.k = L.v = dense_strides(H_kv, Nk, d);
    return fwd_general_impl(q, k, v, o, lse, &L, scale, causal, static_cast<cudaStream_t>(stream));
  }
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
  // at most four query rows per key/value head: the warp-independent kernel (16-key tiles)
  const bool warp_tiles = (H / H_kv) * Lq <= DecWCfg::R;
  if (warp_tiles && !ds->decw_attr) {
    if (cudaFuncSetAttribute(fa_decode_warp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DecWCfg::SMEM_BYTES) != cudaSuccess)
      return FA_ERR_CUDA;
    ds->decw_attr = true;
  }
  CUtensorMap tk, tv;
  const int kt = warp_tiles ? DecWCfg::KT : DecCfg::KT;
  if (!make_map(&tk, k, d, Nk, B * H_kv, kt) || !make_map(&tv, v, d, Nk, B * H_kv, kt)) return FA_ERR_CUDA;
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
  if (warp_tiles)
    fa_decode_warp_kernel<<<grid, DecWCfg::THREADS, DecWCfg::SMEM_BYTES, s>>>(tk, tv, a);
  else if (rows_per_set <= 4)
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
