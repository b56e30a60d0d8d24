// Backward attention kernels for sm_100a (head dim 128).
//
// The backward recomputes the probabilities from Q, K and the saved per-row
// logsumexp instead of reading a stored N x N matrix: the deepfa.ir page
// "Flash Attention: بهینه‌سازی مکانیزم توجه در ترنسفورمرها", section
// "تکنیک 2: محاسبه مجدد" (recomputation), and the nearauto.com FlashAttention-2
// digest, "better parallelism" (in the backward each worker owns a column
// block of the attention matrix, i.e. a block of keys).  The gradient formulas
// are the exact derivative of the forward:
//   P = exp(scale q k - lse),  dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,
//   dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.
//
// Kernels:
//  * fa_bwd_pre_kernel:   D_i, lse_i * log2(e) (padded rows get +inf), dQacc = 0
//  * fa_bwd_kernel:       one CTA per (batch * key/value head, block of 128
//                         keys), looping over blocks of 128 queries (causal: only
//                         those that see the keys) of every query head that reads
//                         this key/value head (one for multi-head attention, a
//                         set of consecutive heads for grouped-query attention, so
//                         dK and dV of the shared head sum over the set in TMEM).  Per query block five 128 x 128 x 128 tcgen05
//                         products:
//                           S^T  = K Q^T           (TMEM X)
//                           dP^T = V dO^T          (TMEM X, once S^T is read out)
//                           dV  += P^T dO          (A = P^T bf16 in TMEM Y)
//                           dQ^T = K^T dS^T        (TMEM Y, after dV)
//                           dK  += dS^T Q          (A = dS^T bf16, smem)
//                         eight warps compute P and dS, two per SM sub-partition
//                         (thread = key row, each warp 64 of the 128 query
//                         columns, all of it elementwise); P goes to the low
//                         half of Y (free once the previous dQ^T half there is
//                         read out), dS to a swizzled [key][query] smem tile;
//                         a warpgroup with one thread per head-dim lane stages
//                         dQ^T in shared memory (in the dO stage the block is
//                         done with) and adds it to the fp32 dQ accumulator
//                         with bulk reductions, 32 query rows at a time;
//  * fa_bwd_dq_kernel:    dQ = bf16(scale * dQacc).
// Sequences, lengths and strides follow layout.cuh (fixed or packed variable
// lengths, bottom-right causal alignment, any row / head / batch strides).
#pragma once

#include "layout.cuh"
#include "ptx.cuh"

namespace fa {

struct BwdArgs {
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;       // indexed by row_index
  float* lse2;            // [B*H][Np] workspace: lse * log2(e), +inf on rows without a query or a key
  float* dvec;            // [B*H][Np] workspace: D_i
  float* dq_acc;          // [acc_rows][D] workspace (fp32), row row_index
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  uint32_t* status;
  SeqLayout L;
  Strides so, sdo, sdq, sdk, sdv;   // element strides of o, dO, dq, dk, dv
  int dq_dense;           // dq is [B][H][Nq][D] dense with fixed lengths (a flat copy of the accumulator)
  int Np;                 // ceil(L.Nq / 128) * 128
  long long acc_rows;     // rows of the dQ accumulator: B*H*Nq, or H*total_q for packed sequences
  int bh_kv;              // B * H_kv (key/value heads); the main kernel's work items
  int group;              // query heads per key/value head
  int n_kb;               // ceil(L.Nk / 128) key blocks
  int heads_per_group;    // work-item order of the main kernel
  int causal;
  float scale;
  float scale_log2;
  unsigned long long wait_limit_ns;
};

// ------------------------------------------------------------------ pre
// D_i = sum_c dO_ic O_ic (bf16 inputs, fp32 sum) and lse_i * log2(e), then the
// fp32 dQ accumulator is zeroed.  HBM-bound: each lane reads 16-byte chunks (a
// row is D / 8 lanes) and a warp keeps U passes of rows in flight before it
// reduces them.
__device__ __forceinline__ float dot_bf16x8(uint4 x, uint4 y) {
  const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 fx = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xs[e]));
    const float2 fy = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ys[e]));
    acc = fmaf(fx.x, fy.x, acc);
    acc = fmaf(fx.y, fy.y, acc);
  }
  return acc;
}

template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const BwdArgs a) {
  constexpr int CPR = D / 8;           // 16-byte chunks per row
  constexpr int RPW = 32 / CPR;        // rows per warp per pass
  constexpr int U = 4;                 // passes in flight
  const int lane = threadIdx.x & 31;
  const int sub = lane / CPR, ch = lane % CPR;
  const long long rows = static_cast<long long>(a.L.B) * a.L.H * a.Np;
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long r0 = gw * (RPW * U); r0 < rows; r0 += nw * (RPW * U)) {   // warp-uniform loop
    uint4 xo[U], xd[U];
    float lv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long r = r0 + u * RPW + sub;
      xo[u] = xd[u] = make_uint4(0u, 0u, 0u, 0u);
      lv[u] = -INFINITY;
      if (r < rows) {
        const int bh = static_cast<int>(r / a.Np);
        const int i = static_cast<int>(r - static_cast<long long>(bh) * a.Np);
        const int b = bh / a.L.H, h = bh - b * a.L.H;
        const SeqSpan sp = seq_span_any(a.L, b, a.status);
        if (i < sp.nq) {
          xo[u] = __ldg(reinterpret_cast<const uint4*>(a.o + row_offset(a.so, sp.bc, h, sp.q0 + i) + ch * 8));
          xd[u] = __ldg(reinterpret_cast<const uint4*>(a.dout + row_offset(a.sdo, sp.bc, h, sp.q0 + i) + ch * 8));
          if (ch == 0) lv[u] = a.lse[row_index_any(a.L, sp, h, i)];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float acc = dot_bf16x8(xo[u], xd[u]);
#pragma unroll
      for (int off = CPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      const long long r = r0 + u * RPW + sub;
      if (ch == 0 && r < rows) {
        // rows past the sequence end, and rows that see no key (lse = -inf), get
        // +inf: their P = 2^(s - inf) is 0
        a.dvec[r] = acc;
        a.lse2[r] = lv[u] == -INFINITY ? INFINITY : lv[u] * 1.4426950408889634f;
      }
    }
  }
  // zero the dQ accumulator
  const size_t n4 = static_cast<size_t>(a.acc_rows) * D / 4;
  float4* q4 = reinterpret_cast<float4*>(a.dq_acc);
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t k = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; k + 3 * stride < n4; k += 4 * stride) {
#pragma unroll
    for (int u = 0; u < 4; ++u) q4[k + u * stride] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (; k < n4; k += stride) q4[k] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ------------------------------------------------------------------ dQ convert
// dQ = bf16(scale * dQacc), four 16-byte loads in flight per thread.
__device__ __forceinline__ uint2 scale_pack4(float4 v, float s) {
  uint2 w;
  w.x = pack_bf16x2(v.x * s, v.y * s);
  w.y = pack_bf16x2(v.z * s, v.w * s);
  return w;
}

template <int D>
__device__ __forceinline__ long long dq_offset(const BwdArgs& a, size_t k) {   // element of dq for float4 k
  const long long ar = static_cast<long long>(k / (D / 4));
  const int c = static_cast<int>(k % (D / 4)) * 4;
  if (a.L.cu_q) {            // [H][total_q]: the row is the packed row coordinate
    const int h = static_cast<int>(ar / a.L.total_q);
    return row_offset(a.sdq, 0, h, static_cast<int>(ar - static_cast<long long>(h) * a.L.total_q)) + c;
  }
  const long long bh = ar / a.L.Nq;  // [B][H][Nq]
  const int b = static_cast<int>(bh / a.L.H);
  return row_offset(a.sdq, b, static_cast<int>(bh - static_cast<long long>(b) * a.L.H),
                    static_cast<int>(ar - bh * a.L.Nq)) + c;
}

template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const BwdArgs a) {
  const size_t n4 = static_cast<size_t>(a.acc_rows) * D / 4;
  const float4* q4 = reinterpret_cast<const float4*>(a.dq_acc);
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t k = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (a.dq_dense) {          // the accumulator's order is dq's
    uint2* out = reinterpret_cast<uint2*>(a.dq);
    for (; k + 3 * stride < n4; k += 4 * stride) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = q4[k + u * stride];
#pragma unroll
      for (int u = 0; u < 4; ++u) out[k + u * stride] = scale_pack4(v[u], a.scale);
    }
    for (; k < n4; k += stride) out[k] = scale_pack4(q4[k], a.scale);
  } else {                   // accumulator row -> (sequence, head, row) -> strided dq
    for (; k + 3 * stride < n4; k += 4 * stride) {
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = q4[k + u * stride];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<uint2*>(a.dq + dq_offset<D>(a, k + u * stride)) = scale_pack4(v[u], a.scale);
    }
    for (; k < n4; k += stride) *reinterpret_cast<uint2*>(a.dq + dq_offset<D>(a, k)) = scale_pack4(q4[k], a.scale);
  }
}

// ------------------------------------------------------------------ main
template <int D_>
struct BwdCfg {
  static constexpr int D = D_;                 // head dim, 64 or 128
  static constexpr int BN = 128;               // keys per CTA
  static constexpr int BM = 128;               // queries per iteration
  static constexpr int THREADS = 448;          // warps 0-7 P/dS, 8-11 dQ drain, 12 MMA, 13 TMA
  static constexpr int PDS_THREADS = 256;
  static constexpr int DRAIN_THREADS = 128;
  // Register split (setmaxnreg).  448 threads launch with 128 registers each
  // (four warps share a sub-partition's 16K registers); P/dS warps take 144,
  // the MMA and TMA warps 112, the drain warps give theirs down to 80:
  // 256 * 144 + 128 * 80 + 64 * 112 = 54272 <= 448 * 128, and per sub-partition
  // 2 * 144 + 80 + 112 = 480 <= 512 registers per thread slot.  setmaxnreg.inc
  // draws on registers freed in its own sub-partition, so each must free what its
  // warps take: sub-partitions 2 and 3 hold two P/dS warps (+16 each) and one
  // drain warp (-48); a split that does not balance there waits forever.
  static constexpr int LAUNCH_REGS = 128;
  static constexpr int REGS_PDS = 144, REGS_DRAIN = 80, REGS_SINGLE = 112;
  static constexpr int REG = 128 * 128;        // one 64-column SW128 region of a 128-row bf16 tile
  static constexpr int N_REG = D / 64;         // regions of a 128-row, D-column tile
  static constexpr int TILE = N_REG * REG;     // a 128 x D bf16 tile (K, V, Q or dO)
  static constexpr int DS_BYTES = 2 * REG;     // the 128 x 128 dS tile
  static constexpr int CHUNK_FLOATS = 32 * D;  // 32 query rows of fp32 dQ; two fill a dO stage
  static constexpr int OFF_K = 0, OFF_V = TILE;
  static constexpr int OFF_Q = 2 * TILE;       // two Q stages
  static constexpr int OFF_DO = 4 * TILE;      // two dO stages
  static constexpr int OFF_PS = 6 * TILE;      // dS_i, stored [key][query]
  static constexpr int OFF_VEC = OFF_PS + DS_BYTES;   // per Q stage: lse2[BM] then D[BM]
  static constexpr int VEC_BYTES = 2 * BM * 4;
  static constexpr int OFF_BAR = OFF_VEC + 2 * VEC_BYTES;
  static constexpr int N_BARS = 20;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int USED = OFF_MISC + 16;
  // At most the opt-in maximum per block.  The kernel rounds its base up to 1 KB
  // (SW128 tiles) inside this and checks that USED still fits.
  static constexpr int SMEM_BYTES = (USED + 1024 < 232448) ? USED + 1024 : 232448;
  static constexpr uint32_t TMEM_COLS = 512;
  // X: S^T, then dP^T.  Y: P^T (bf16, columns 0-63), then dQ^T (fp32, 128 columns;
  // with D = 64 the MMA still writes 128 rows of dQ^T, of which lanes >= 64 read
  // the tile after K and are never drained)
  static constexpr uint32_t T_DV = 0, T_DK = D, T_X = 2 * D, T_Y = 2 * D + 128;
  static constexpr uint32_t IDESC_SD = idesc_bf16_f32(128, BM, false, false);   // S^T, dP^T
  static constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, D, false, true);     // dV (A in TMEM), dK
  static constexpr uint32_t IDESC_Q = idesc_bf16_f32(128, BM, true, true);      // dQ^T
};
static_assert(BwdCfg<128>::USED + 768 <= BwdCfg<128>::SMEM_BYTES, "shared memory plan");
static_assert(2 * BwdCfg<128>::CHUNK_FLOATS * 4 == BwdCfg<128>::TILE && 2 * BwdCfg<64>::CHUNK_FLOATS * 4 == BwdCfg<64>::TILE,
              "two dQ chunks fill one dO stage");
static_assert(BwdCfg<64>::USED + 768 <= BwdCfg<64>::SMEM_BYTES, "shared memory plan");
static_assert(BwdCfg<128>::PDS_THREADS * BwdCfg<128>::REGS_PDS + BwdCfg<128>::DRAIN_THREADS * BwdCfg<128>::REGS_DRAIN +
                  64 * BwdCfg<128>::REGS_SINGLE <= BwdCfg<128>::THREADS * BwdCfg<128>::LAUNCH_REGS,
              "register split exceeds the registers the block launches with");
static_assert(2 * BwdCfg<128>::REGS_PDS + BwdCfg<128>::REGS_DRAIN + BwdCfg<128>::REGS_SINGLE <= 512,
              "register split exceeds a sub-partition");
static_assert(2 * (BwdCfg<128>::REGS_PDS - BwdCfg<128>::LAUNCH_REGS) <=
                  BwdCfg<128>::LAUNCH_REGS - BwdCfg<128>::REGS_DRAIN,
              "register split does not balance within a sub-partition");

// Work item x -> (head, key block).  Heads are taken in groups of
// heads_per_group; inside a group the key blocks with the most query blocks
// come first (causal), so the dQ accumulators being added to at any time are
// those of a few heads and stay in L2.
__host__ __device__ __forceinline__ void bwd_decode(const BwdArgs& a, int x, int& bh, int& kb) {   // bh: b * H_kv + h_kv
  const int per_group = a.heads_per_group * a.n_kb;
  const int g = x / per_group;
  const int r = x - g * per_group;
  const int h0 = g * a.heads_per_group;
  const int gh = min(a.heads_per_group, a.bh_kv - h0);
  kb = r / gh;
  bh = h0 + (r - kb * gh);
}

template <int D_, bool PACKED>
__global__ void __launch_bounds__(BwdCfg<D_>::THREADS, 1)
fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const BwdArgs args) {
  using C = BwdCfg<D_>;
  constexpr int D = C::D;
  extern __shared__ __align__(16) uint8_t smem_raw[];   // only 16 B promised: the 1 KB rounding below is real
  int bh, kb;                                        // bh: key/value head (b * H_kv + h_kv)
  bwd_decode(args, static_cast<int>(blockIdx.x), bh, kb);
  const int b = bh / args.L.H_kv, h_kv = bh - b * args.L.H_kv;
  const SeqSpan sp = seq_span<PACKED>(args.L, b, args.status);
  const int k0 = kb * C::BN;                         // first key of the block, in the sequence
  if (k0 >= sp.nk) return;                           // past this sequence's keys: nothing to do
  const int off = sp.nk - sp.nq;                     // bottom-right causal alignment
  const int n_qb = (sp.nq + C::BM - 1) / C::BM;
  // query blocks that see these keys (every key is seen by the last query row)
  const int i_begin = args.causal ? max(0, k0 - off) / C::BM : 0;
  const int n_per = max(0, n_qb - i_begin);          // per query head
  const int n_iter = n_per * args.group;             // every query head of the set, one after the other
  if (n_iter == 0) {                                 // no query at all: dK = dV = 0
    const int nk = min(C::BN, sp.nk - k0);
    for (int e = threadIdx.x; e < nk * (D / 8); e += blockDim.x) {
      const int r = e / (D / 8), c = (e % (D / 8)) * 8;
      *reinterpret_cast<uint4*>(args.dk + row_offset(args.sdk, sp.bc, h_kv, sp.k0 + k0 + r) + c) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(args.dv + row_offset(args.sdv, sp.bc, h_kv, sp.k0 + k0 + r) + c) = make_uint4(0, 0, 0, 0);
    }
    return;
  }
  // query head (in the batch entry) and query block of iteration it
  auto q_head = [&](int it) { return h_kv * args.group + it / n_per; };
  auto q_row0 = [&](int it) { return (i_begin + it % n_per) * C::BM; };
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  if (pad + C::USED > static_cast<uint32_t>(C::SMEM_BYTES)) {   // buffers do not fit: report, touch nothing
    if (threadIdx.x == 0) atomicOr(args.status, DEV_SMEM);
    return;
  }
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V, sPS = sbase + C::OFF_PS;
  auto sQ = [&](int s) { return sbase + C::OFF_Q + s * C::TILE; };
  auto sDO = [&](int s) { return sbase + C::OFF_DO + s * C::TILE; };
  auto sVec = [&](int s) { return sbase + C::OFF_VEC + s * C::VEC_BYTES; };
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  const uint32_t b_kv_full = bar(0);
  auto b_q_full = [&](int s) { return bar(1 + s); };
  auto b_q_empty = [&](int s) { return bar(3 + s); };
  auto b_do_full = [&](int s) { return bar(5 + s); };
  auto b_do_empty = [&](int s) { return bar(7 + s); };
  const uint32_t b_s_full = bar(9);      // S_i in X
  const uint32_t b_dp_full = bar(10);    // dP_i in X
  const uint32_t b_x_free = bar(11);     // X read out (twice per query block: S, then dP)
  const uint32_t b_p_ready = bar(12);    // P_i in the low half of Y
  const uint32_t b_ylo_free = bar(13);   // low half of Y read out (dQ^T_i, queries 0-63)
  const uint32_t b_ds_ready = bar(14);   // dS_i in the dS tile
  const uint32_t b_ps_free = bar(15);    // dQ_i, dK_i done reading dS_i
  const uint32_t b_dq_full = bar(16);    // dQ^T_i in Y
  const uint32_t b_yhi_free = bar(17);   // all of Y read out
  const uint32_t b_dkv_done = bar(18);
  const uint32_t b_drain = bar(19);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *abort_flag = 0u;
    mbar_init(b_kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(b_q_full(s), 1);
      mbar_init(b_q_empty(s), 1);
      mbar_init(b_do_full(s), 1);
      mbar_init(b_do_empty(s), 1);
    }
    mbar_init(b_s_full, 1);
    mbar_init(b_dp_full, 1);
    mbar_init(b_x_free, C::PDS_THREADS);
    mbar_init(b_p_ready, C::PDS_THREADS);
    mbar_init(b_ylo_free, C::DRAIN_THREADS);
    mbar_init(b_ds_ready, C::PDS_THREADS);
    mbar_init(b_ps_free, 1);
    mbar_init(b_dq_full, 1);
    mbar_init(b_yhi_free, C::DRAIN_THREADS);
    mbar_init(b_dkv_done, 1);
    mbar_init(b_drain, 1);
    fence_mbar_init();
  }
  if (warp == 12) tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
  if (warp == 13 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, args.status, args.wait_limit_ns};

  if (warp == 13) {
    // ------------------------------------------------------------ TMA producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 112;");
    if (lane == 0) {
      bool ok = true;
      int q_last[2] = {-1, -1}, do_last[2] = {-1, -1};     // last query block loaded into each stage
      mbar_expect_tx(b_kv_full, 2 * C::TILE);
      for (int r = 0; r < C::N_REG; ++r) {
        tma_load_4d(sK + r * C::REG, &tm_k, b_kv_full, r * 64, sp.k0 + k0, h_kv, sp.bc);
        tma_load_4d(sV + r * C::REG, &tm_v, b_kv_full, r * 64, sp.k0 + k0, h_kv, sp.bc);
      }
      for (int it = 0; it < n_iter; ++it) {
        const int s = it & 1;
        const uint32_t round = static_cast<uint32_t>(it) >> 1;
        const int q0 = q_row0(it);
        const int hq = q_head(it);
        // Q_i with its lse2 and D rows; the stage is released after dK_i
        if (round > 0 && !mbar_wait(b_q_empty(s), (round - 1) & 1, ctl)) { ok = false; break; }
        mbar_expect_tx(b_q_full(s), C::TILE + C::VEC_BYTES);
        for (int r = 0; r < C::N_REG; ++r)
          tma_load_4d(sQ(s) + r * C::REG, &tm_q, b_q_full(s), r * 64, sp.q0 + q0, hq, sp.bc);
        const size_t voff = (static_cast<size_t>(b) * args.L.H + hq) * args.Np + q0;
        bulk_load(sVec(s), args.lse2 + voff, C::BM * 4, b_q_full(s));
        bulk_load(sVec(s) + C::BM * 4, args.dvec + voff, C::BM * 4, b_q_full(s));
        q_last[s] = it;
        // dO_i; the stage is released after dV_i
        if (round > 0 && !mbar_wait(b_do_empty(s), (round - 1) & 1, ctl)) { ok = false; break; }
        mbar_expect_tx(b_do_full(s), C::TILE);
        for (int r = 0; r < C::N_REG; ++r)
          tma_load_4d(sDO(s) + r * C::REG, &tm_do, b_do_full(s), r * 64, sp.q0 + q0, hq, sp.bc);
        do_last[s] = it;
      }
      if (!ok) {       // let the loads in flight land before the CTA exits
        mbar_wait_quiet(b_kv_full, 0, 200000000ull);
        for (int s = 0; s < 2; ++s) {
          if (q_last[s] >= 0) mbar_wait_quiet(b_q_full(s), (q_last[s] >> 1) & 1, 200000000ull);
          if (do_last[s] >= 0) mbar_wait_quiet(b_do_full(s), (do_last[s] >> 1) & 1, 200000000ull);
        }
      }
    }
  } else if (warp == 12) {
    // ------------------------------------------------------------ MMA issuer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 112;");
    if (lane == 0) {
      // Descriptors are built once; a K step adds to the start-address field:
      // K-major tiles advance 32 B inside a 128-B row and switch region every
      // four steps, MN-major tiles advance 16 rows (2 KB).
      const uint64_t dK_k = sdesc_sw128(sK, 16, 1024), dV_k = sdesc_sw128(sV, 16, 1024);
      const uint64_t dK_mn = sdesc_sw128(sK, C::REG, 1024);
      const uint64_t dPS_k = sdesc_sw128(sPS, 16, 1024), dPS_mn = sdesc_sw128(sPS, C::REG, 1024);
      const uint64_t dQ_k0 = sdesc_sw128(sQ(0), 16, 1024), dQ_k1 = sdesc_sw128(sQ(1), 16, 1024);
      const uint64_t dQ_mn0 = sdesc_sw128(sQ(0), C::REG, 1024), dQ_mn1 = sdesc_sw128(sQ(1), C::REG, 1024);
      const uint64_t dO_k0 = sdesc_sw128(sDO(0), 16, 1024), dO_k1 = sdesc_sw128(sDO(1), 16, 1024);
      const uint64_t dO_mn0 = sdesc_sw128(sDO(0), C::REG, 1024), dO_mn1 = sdesc_sw128(sDO(1), C::REG, 1024);
      auto kstep = [](int kk) { return static_cast<uint64_t>((kk >> 2) * (C::REG >> 4) + (kk & 3) * 2); };
      auto mnstep = [](int kk) { return static_cast<uint64_t>(kk * (2048 >> 4)); };
      // S^T = K Q^T and dP^T = V dO^T (both operands K-major), into X
      auto issue_kmaj = [&](uint64_t a, uint64_t b) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) umma_ss(tmem + C::T_X, a + kstep(kk), b + kstep(kk), C::IDESC_SD, kk > 0);
      };
      // dV += P^T dO (A = P^T in Y, 8 packed columns per K step), dK += dS^T Q
      // (A = the dS tile, K-major); B MN-major
      auto issue_dv = [&](uint64_t b, bool acc) {
#pragma unroll
        for (int kk = 0; kk < C::BM / 16; ++kk)
          umma_ts(tmem + C::T_DV, tmem + C::T_Y + 8 * kk, b + mnstep(kk), C::IDESC_KV, (acc || kk > 0) ? 1u : 0u);
      };
      auto issue_dk = [&](uint64_t b, bool acc) {
#pragma unroll
        for (int kk = 0; kk < C::BM / 16; ++kk)
          umma_ss(tmem + C::T_DK, dPS_k + kstep(kk), b + mnstep(kk), C::IDESC_KV, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(b_kv_full, 0, ctl);
      // prologue: S_0, and dP_0 once S_0 has been read out of X
      if (ok) ok = mbar_wait(b_q_full(0), 0, ctl);
      if (ok) {
        tc_fence_after();
        issue_kmaj(dK_k, dQ_k0);
        umma_commit(b_s_full);
        ok = mbar_wait(b_x_free, 0, ctl) && mbar_wait(b_do_full(0), 0, ctl);
      }
      if (ok) {
        tc_fence_after();
        issue_kmaj(dV_k, dO_k0);
        umma_commit(b_dp_full);
      }
      for (int it = 0; it < n_iter && ok; ++it) {
        const int s = it & 1;
        const uint32_t ph = static_cast<uint32_t>(it) & 1;
        const bool more = it + 1 < n_iter;
        const uint32_t ph1 = (static_cast<uint32_t>(it + 1) >> 1) & 1;   // round parity of block it + 1
        // dV += P_i^T dO_i
        if (!mbar_wait(b_p_ready, ph, ctl)) { ok = false; break; }
        tc_fence_after();
        issue_dv(s ? dO_mn1 : dO_mn0, it > 0);   // the dO stage is released by the dQ drain
        // S_{i+1}, once dP_i has been read out of X
        if (more) {
          if (!mbar_wait(b_x_free, 1, ctl) || !mbar_wait(b_q_full(s ^ 1), ph1, ctl)) { ok = false; break; }
          tc_fence_after();
          issue_kmaj(dK_k, s ? dQ_k0 : dQ_k1);
          umma_commit(b_s_full);
        }
        // dQ^T_i = K^T dS_i^T (into Y, after dV_i has read P_i there), then dK += dS_i^T Q_i
        if (!mbar_wait(b_ds_ready, ph, ctl)) { ok = false; break; }
        if (it > 0 && !mbar_wait(b_yhi_free, ph ^ 1u, ctl)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          umma_ss(tmem + C::T_Y, dK_mn + mnstep(kk), dPS_mn + mnstep(kk), C::IDESC_Q, kk > 0);
        umma_commit(b_dq_full);
        issue_dk(s ? dQ_mn1 : dQ_mn0, it > 0);
        umma_commit(b_q_empty(s));
        umma_commit(b_ps_free);
        // dP_{i+1}, once S_{i+1} has been read out of X
        if (more) {
          if (!mbar_wait(b_x_free, 0, ctl) || !mbar_wait(b_do_full(s ^ 1), ph1, ctl)) { ok = false; break; }
          tc_fence_after();
          issue_kmaj(dV_k, s ? dO_k0 : dO_k1);
          umma_commit(b_dp_full);
        }
      }
      if (ok) umma_commit(b_dkv_done);
      umma_commit(b_drain);
      mbar_wait_quiet(b_drain, 0, 200000000ull);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ P / dS warps (thread = key, 64 query columns)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 144;");
    const int quarter = warp & 3;
    const int ch = warp >> 2;                       // which 64 of the 128 query columns
    const int rloc = quarter * 32 + lane;           // key row in the block == TMEM lane
    const int key = k0 + rloc;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tX = tmem + lane_off + C::T_X + 64 * ch;
    const uint32_t tP = tmem + lane_off + C::T_Y + 32 * ch;     // this thread's 64 P values, packed
    const float c2 = args.scale_log2;
    const bool key_ok = key < sp.nk;
    // this thread's half row of the dS tile: region ch, row rloc; 16-byte
    // chunk j of the row sits at chunk j ^ (row & 7) (128-byte swizzle)
    uint8_t* prow = smem + C::OFF_PS + ch * C::REG + rloc * 128;
    const int sw = rloc & 7;
    bool ok = true;
    for (int it = 0; it < n_iter; ++it) {
      const int s = it & 1;
      const uint32_t ph = static_cast<uint32_t>(it) & 1;
      const int q0 = q_row0(it);
      const float* lse2 = reinterpret_cast<const float*>(smem + C::OFF_VEC + s * C::VEC_BYTES) + 64 * ch;
      const float* dvec = lse2 + C::BM;
      if (!mbar_wait_warp(b_q_full(s), (static_cast<uint32_t>(it) >> 1) & 1, ctl)) { ok = false; break; }
      if (!mbar_wait_warp(b_s_full, ph, ctl)) { ok = false; break; }
      tc_fence_after();
      float p[64];
      {
        uint32_t ra[32], rb[32];
        tmem_ld32(tX, ra);
        tmem_ld32(tX + 32, rb);
        tmem_wait_ld();
        reg_fence32(ra);
        reg_fence32(rb);
        tc_fence_before();
        mbar_arrive(b_x_free);
        // 2^x: three pairs in eight on the FMA pipe (ex2_poly2), the rest on the
        // special-function unit, which would otherwise be the limit here
        const float2 c2v = make_float2(c2, c2);
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float2 la = *reinterpret_cast<const float2*>(lse2 + c);
          const float2 lb = *reinterpret_cast<const float2*>(lse2 + 32 + c);
          const float2 xa = ffma2(make_float2(__uint_as_float(ra[c]), __uint_as_float(ra[c + 1])), c2v,
                                  make_float2(-la.x, -la.y));
          const float2 xb = ffma2(make_float2(__uint_as_float(rb[c]), __uint_as_float(rb[c + 1])), c2v,
                                  make_float2(-lb.x, -lb.y));
          if ((0x92u >> ((c >> 1) & 7)) & 1u) {
            const float2 ea = ex2_poly2(xa), eb = ex2_poly2(xb);
            p[c] = ea.x;
            p[c + 1] = ea.y;
            p[32 + c] = eb.x;
            p[32 + c + 1] = eb.y;
          } else {
            p[c] = ex2_approx(xa.x);
            p[c + 1] = ex2_approx(xa.y);
            p[32 + c] = ex2_approx(xb.x);
            p[32 + c + 1] = ex2_approx(xb.y);
          }
        }
      }
      // keys past the sequence end, and (causal) queries that do not see this key, get P = 0
      const int cut = !key_ok ? C::BM : (args.causal ? key - off - q0 : 0);   // columns c < cut are masked
      if (cut > 64 * ch) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (64 * ch + c < cut) p[c] = 0.f;
      }
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) pk[c] = pack_bf16x2(p[2 * c], p[2 * c + 1]);
      // P^T into the low half of Y, once the previous dQ^T there has been read out
      if (it > 0 && !mbar_wait_warp(b_ylo_free, ph ^ 1u, ctl)) { ok = false; break; }
      tc_fence_after();
      tmem_st32(tP, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(b_p_ready);
      // dS = P (dP - D)
      if (!mbar_wait_warp(b_dp_full, ph, ctl)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {      // two 32-column halves (register budget)
        uint32_t ra[32];
        tmem_ld32(tX + 32 * h, ra);
        tmem_wait_ld();
        reg_fence32(ra);
        if (h == 1) {
          tc_fence_before();
          mbar_arrive(b_x_free);
        }
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float2 dd = *reinterpret_cast<const float2*>(dvec + 32 * h + c);
          const float2 g = fmul2(make_float2(p[32 * h + c], p[32 * h + c + 1]),
                                 fsub2(make_float2(__uint_as_float(ra[c]), __uint_as_float(ra[c + 1])), dd));
          pk[16 * h + (c >> 1)] = pack_bf16x2(g.x, g.y);
        }
      }
      if (it > 0 && !mbar_wait_warp(b_ps_free, ph ^ 1u, ctl)) { ok = false; break; }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint4*>(prow + ((j ^ sw) << 4)) = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      fence_proxy_async_smem();
      mbar_arrive(b_ds_ready);
    }
    // ---- epilogue: this thread's half of the dV, dK rows (D / 2 columns) -> global
    if (ok && mbar_wait_warp(b_dkv_done, 0, ctl)) {
      tc_fence_after();
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t tsrc = tmem + lane_off + (which ? C::T_DK : C::T_DV) + (D / 2) * ch;
        __nv_bfloat16* dst = which ? args.dk + row_offset(args.sdk, sp.bc, h_kv, sp.k0 + key) + (D / 2) * ch
                                   : args.dv + row_offset(args.sdv, sp.bc, h_kv, sp.k0 + key) + (D / 2) * ch;
        const float mul = which ? args.scale : 1.0f;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t v[32];
          tmem_ld32(tsrc + c * 32, v);
          tmem_wait_ld();
          reg_fence32(v);
          if (key_ok) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(v[8 * e + 0]) * mul, __uint_as_float(v[8 * e + 1]) * mul);
              w.y = pack_bf16x2(__uint_as_float(v[8 * e + 2]) * mul, __uint_as_float(v[8 * e + 3]) * mul);
              w.z = pack_bf16x2(__uint_as_float(v[8 * e + 4]) * mul, __uint_as_float(v[8 * e + 5]) * mul);
              w.w = pack_bf16x2(__uint_as_float(v[8 * e + 6]) * mul, __uint_as_float(v[8 * e + 7]) * mul);
              d4[e] = w;
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ dQ drain (thread = head-dim lane)
    // dQ^T_i leaves tensor memory in four 32-query chunks.  Each chunk is
    // written row-major ([query][d], fp32) into one half of the dO stage block i
    // has finished with (dP^T_i and dV_i, its only readers, completed before
    // dQ^T_i), and one thread adds it to the accumulator with a bulk reduction:
    // whole lines from one instruction instead of a scalar atomic per element.
    // The stage goes back to the loader once the reductions have read it.
    // The wait for each block ends in a vote of the four drain warps, so they
    // leave together and none is left at a later named barrier.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 80;");
    const int dl = (warp - 8) * 32 + lane;
    const bool issuer = dl == 0;
    const uint32_t tY = tmem + (static_cast<uint32_t>((warp - 8) * 32) << 16) + C::T_Y;
    for (int it = 0; it < n_iter; ++it) {
      const int s = it & 1;
      if (!named_bar_and(1, C::DRAIN_THREADS, mbar_wait_warp(b_dq_full, static_cast<uint32_t>(it) & 1, ctl))) break;
      tc_fence_after();
      const int q0 = q_row0(it);
      const int nq = min(C::BM, sp.nq - q0);
      float* stage = reinterpret_cast<float*>(smem + C::OFF_DO + s * C::TILE);
#pragma unroll
      for (int c = 0; c < 4; ++c) {      // chunk c: queries 32c .. 32c + 31 of the block
        uint32_t r[32];
        tmem_ld32(tY + 32 * c, r);
        tmem_wait_ld();
        reg_fence32(r);
        if (c & 1) {                     // a 64-column half of Y read out: P (low) or dQ^T_{i+1} may go there
          tc_fence_before();
          mbar_arrive(c == 1 ? b_ylo_free : b_yhi_free);
        }
        const int rows = min(32, nq - 32 * c);       // uniform over the drain warps; later chunks have fewer
        if (rows <= 0) continue;
        if (c >= 2) {                                // chunk c - 2 has been read out of this buffer
          if (issuer) bulk_wait_read<1>();
          named_bar_sync(1, C::DRAIN_THREADS);
        }
        float* buf = stage + (c & 1) * C::CHUNK_FLOATS;
        if (dl < D) {                                // none for the lanes past the head dim (D = 64)
#pragma unroll
          for (int j = 0; j < 32; ++j) buf[j * D + dl] = __uint_as_float(r[j]);
        }
        fence_proxy_async_smem();
        named_bar_sync(1, C::DRAIN_THREADS);
        if (issuer) {
          float* acc = args.dq_acc + (row_index<PACKED>(args.L, sp, q_head(it), q0) + 32 * c) * D;
          bulk_reduce_add_f32(acc, sDO(s) + (c & 1) * C::CHUNK_FLOATS * 4, static_cast<uint32_t>(rows) * D * 4);
          bulk_commit();
        }
      }
      if (issuer) {
        bulk_wait_read<0>();
        mbar_arrive(b_do_empty(s));
      }
    }
    if (issuer) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
