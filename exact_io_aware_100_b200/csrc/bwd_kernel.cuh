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
//  * fa_bwd_kernel:       one CTA per (batch*head, block of 128 keys), looping
//                         over blocks of 64 queries (causal: only those that see
//                         the keys).  Per query block five tcgen05 MMAs:
//                           S^T  = K Q^T           (TMEM, 64 cols)
//                           dP^T = V dO^T          (TMEM, 64 cols)
//                           dV  += P^T dO          (A = P^T bf16 from TMEM)
//                           dK  += dS^T Q          (A = dS^T bf16 from TMEM)
//                           dQ^T = K^T dS^T        (both operands MN-major smem)
//                         eight warps compute P and dS, two per SM sub-partition
//                         (thread = key row, each warp 32 of the 64 query columns,
//                         all of it elementwise); a warpgroup with one thread per
//                         head-dim lane drains dQ^T into the fp32 dQ accumulator
//                         with atomic adds;
//  * fa_bwd_dq_kernel:    dQ = bf16(scale * dQacc).
#pragma once

#include "ptx.cuh"

namespace fa {

struct BwdArgs {
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;       // [BH, N]
  float* lse2;            // [BH, Np] workspace: lse * log2(e), +inf on padded rows
  float* dvec;            // [BH, Np] workspace: D_i
  float* dq_acc;          // [BH, N, D] workspace (fp32)
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  uint32_t* status;
  int N, Np, bh;
  int n_kb;               // ceil(N / 128)
  int n_qb;               // ceil(N / 64)
  int causal;
  float scale;
  float scale_log2;
  unsigned long long wait_limit_ns;
};

// ------------------------------------------------------------------ pre
// One warp per query row: D_i = sum_c dO_ic O_ic (bf16 inputs, fp32 sum).
template <int D>
__global__ void fa_bwd_pre_kernel(const BwdArgs a) {
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(a.bh) * a.Np;
  for (long long r = gw; r < rows; r += warps) {
    const int bh = static_cast<int>(r / a.Np);
    const int i = static_cast<int>(r % a.Np);
    float acc = 0.f;
    if (i < a.N) {
      const size_t base = (static_cast<size_t>(bh) * a.N + i) * D;
      constexpr int PER = D / 32;        // elements per lane
      const __nv_bfloat16* po = a.o + base + lane * PER;
      const __nv_bfloat16* pd = a.dout + base + lane * PER;
#pragma unroll
      for (int e = 0; e < PER; e += 2) {
        const float2 fo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(po + e));
        const float2 fd = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(pd + e));
        acc = fmaf(fo.x, fd.x, acc);
        acc = fmaf(fo.y, fd.y, acc);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      a.dvec[r] = acc;
      a.lse2[r] = (i < a.N) ? a.lse[static_cast<size_t>(bh) * a.N + i] * 1.4426950408889634f : INFINITY;
    }
  }
  // zero the dQ accumulator
  const size_t n4 = static_cast<size_t>(a.bh) * a.N * D / 4;
  float4* q4 = reinterpret_cast<float4*>(a.dq_acc);
  for (size_t k = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; k < n4;
       k += static_cast<size_t>(gridDim.x) * blockDim.x)
    q4[k] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ------------------------------------------------------------------ dQ convert
template <int D>
__global__ void fa_bwd_dq_kernel(const BwdArgs a) {
  const size_t n4 = static_cast<size_t>(a.bh) * a.N * D / 4;
  const float4* q4 = reinterpret_cast<const float4*>(a.dq_acc);
  uint2* out = reinterpret_cast<uint2*>(a.dq);
  for (size_t k = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; k < n4;
       k += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 v = q4[k];
    uint2 w;
    w.x = pack_bf16x2(v.x * a.scale, v.y * a.scale);
    w.y = pack_bf16x2(v.z * a.scale, v.w * a.scale);
    out[k] = w;
  }
}

// ------------------------------------------------------------------ main
struct BwdCfg {
  static constexpr int D = 128;
  static constexpr int BN = 128;               // keys per CTA
  static constexpr int BM = 64;                // queries per iteration
  static constexpr int STAGES = 3;
  static constexpr int THREADS = 448;          // warps 0-7 P/dS, 8-11 dQ drain, 12 MMA, 13 TMA
  static constexpr int PDS_THREADS = 256;
  static constexpr int KREG = 128 * 128;       // 64-col region of a 128-row tile
  static constexpr int QREG = 64 * 128;        // 64-col region of a 64-row tile
  static constexpr int KV_TILE = BN * D * 2;   // 32 KB
  static constexpr int Q_TILE = BM * D * 2;    // 16 KB
  static constexpr int ST_Q = 0, ST_DO = Q_TILE, ST_LSE = 2 * Q_TILE, ST_DV = 2 * Q_TILE + BM * 4;
  static constexpr int STAGE_BYTES = 2 * Q_TILE + 2 * BM * 4;    // 33280
  static constexpr int STAGE_STRIDE = 33792;                     // next multiple of 1024
  static constexpr int DS_BYTES = BN * BM * 2;                   // 16 KB
  static constexpr int OFF_K = 0, OFF_V = KV_TILE, OFF_ST = 2 * KV_TILE;
  static constexpr int OFF_DS = OFF_ST + STAGES * STAGE_STRIDE;
  static constexpr int OFF_BAR = OFF_DS + 2 * DS_BYTES;
  // barriers: kv_full, qdo_full[S], qdo_empty[S], s_full, dp_full, p_full, ds_full,
  //           dq_full[2], dq_free[2], dkv_done, drain
  static constexpr int N_BARS = 1 + 2 * STAGES + 4 + 4 + 2;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_DV = 0, T_DK = 128, T_S = 256, T_DP = 320, T_DQ = 384;
  static constexpr uint32_t IDESC_SD = idesc_bf16_f32(128, BM, false, false);   // S^T, dP^T
  static constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, D, false, true);     // dV, dK
  static constexpr uint32_t IDESC_Q = idesc_bf16_f32(128, BM, true, true);      // dQ^T
};

__global__ void __launch_bounds__(BwdCfg::THREADS, 1)
fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const BwdArgs args) {
  using C = BwdCfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V;
  auto sStage = [&](int s) { return sbase + C::OFF_ST + s * C::STAGE_STRIDE; };
  auto sDS = [&](int b) { return sbase + C::OFF_DS + b * C::DS_BYTES; };
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t b_kv_full = bar0;
  auto b_qdo_full = [&](int s) { return bar0 + 8 + 8 * s; };
  auto b_qdo_empty = [&](int s) { return bar0 + 8 + 8 * C::STAGES + 8 * s; };
  const uint32_t b_s_full = bar0 + 8 + 16 * C::STAGES;
  const uint32_t b_dp_full = b_s_full + 8;
  const uint32_t b_p_full = b_s_full + 16;
  const uint32_t b_ds_full = b_s_full + 24;
  auto b_dq_full = [&](int b) { return b_s_full + 32 + 8 * b; };
  auto b_dq_free = [&](int b) { return b_s_full + 48 + 8 * b; };
  const uint32_t b_dkv_done = b_s_full + 64;
  const uint32_t b_drain = b_s_full + 72;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // work item: key blocks with the most query blocks first (causal), then heads
  const int kb = static_cast<int>(blockIdx.x) / args.bh;
  const int bh = static_cast<int>(blockIdx.x) % args.bh;
  const int k0 = kb * C::BN;
  const int i_begin = args.causal ? (k0 / C::BM) : 0;
  const int n_iter = args.n_qb - i_begin;

  if (threadIdx.x == 0) {
    *abort_flag = 0u;
    mbar_init(b_kv_full, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(b_qdo_full(s), 1);
      mbar_init(b_qdo_empty(s), 1);
    }
    mbar_init(b_s_full, 1);
    mbar_init(b_dp_full, 1);
    mbar_init(b_p_full, C::PDS_THREADS);
    mbar_init(b_ds_full, C::PDS_THREADS);
    for (int b = 0; b < 2; ++b) {
      mbar_init(b_dq_full(b), 1);
      mbar_init(b_dq_free(b), 128);
    }
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
    if (lane == 0) {
      bool ok = true;
      uint32_t issued = 0, last_parity = 0;      // per-stage bit masks
      mbar_expect_tx(b_kv_full, 2 * C::KV_TILE);
      for (int r = 0; r < 2; ++r) {
        tma_load_3d(sK + r * C::KREG, &tm_k, b_kv_full, r * 64, k0, bh);
        tma_load_3d(sV + r * C::KREG, &tm_v, b_kv_full, r * 64, k0, bh);
      }
      for (int it = 0; it < n_iter; ++it) {
        const int s = it % C::STAGES;
        const uint32_t round = it / C::STAGES;
        if (round > 0 && !mbar_wait(b_qdo_empty(s), (round - 1) & 1, ctl)) { ok = false; break; }
        const int q0 = (i_begin + it) * C::BM;
        const uint32_t st = sStage(s);
        mbar_expect_tx(b_qdo_full(s), C::STAGE_BYTES);
        for (int r = 0; r < 2; ++r) {
          tma_load_3d(st + C::ST_Q + r * C::QREG, &tm_q, b_qdo_full(s), r * 64, q0, bh);
          tma_load_3d(st + C::ST_DO + r * C::QREG, &tm_do, b_qdo_full(s), r * 64, q0, bh);
        }
        const size_t voff = static_cast<size_t>(bh) * args.Np + q0;
        bulk_load(st + C::ST_LSE, args.lse2 + voff, C::BM * 4, b_qdo_full(s));
        bulk_load(st + C::ST_DV, args.dvec + voff, C::BM * 4, b_qdo_full(s));
        issued |= 1u << s;
        last_parity = (last_parity & ~(1u << s)) | ((round & 1u) << s);
      }
      if (!ok) {
        mbar_wait_quiet(b_kv_full, 0, 200000000ull);
        for (int s = 0; s < C::STAGES; ++s)
          if ((issued >> s) & 1u) mbar_wait_quiet(b_qdo_full(s), (last_parity >> s) & 1u, 200000000ull);
      }
    }
  } else if (warp == 12) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(b_kv_full, 0, ctl);
      tc_fence_after();
      auto issue_s = [&](int s) {       // S^T = K Q^T
        const uint32_t qb = sStage(s) + C::ST_Q;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * C::KREG + (kk & 3) * 32;
          const uint32_t qo = (kk >> 2) * C::QREG + (kk & 3) * 32;
          umma_ss(tmem + C::T_S, sdesc_sw128(sK + ko, 16, 1024), sdesc_sw128(qb + qo, 16, 1024),
                  C::IDESC_SD, kk > 0);
        }
        umma_commit(b_s_full);
      };
      auto issue_dp = [&](int s) {      // dP^T = V dO^T
        const uint32_t db = sStage(s) + C::ST_DO;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * C::KREG + (kk & 3) * 32;
          const uint32_t qo = (kk >> 2) * C::QREG + (kk & 3) * 32;
          umma_ss(tmem + C::T_DP, sdesc_sw128(sV + ko, 16, 1024), sdesc_sw128(db + qo, 16, 1024),
                  C::IDESC_SD, kk > 0);
        }
        umma_commit(b_dp_full);
      };
      if (ok) {
        if (!mbar_wait(b_qdo_full(0), 0, ctl)) ok = false;
        tc_fence_after();
      }
      if (ok) {
        issue_s(0);
        issue_dp(0);
      }
      for (int it = 0; it < n_iter && ok; ++it) {
        const int s = it % C::STAGES;
        const uint32_t ph = it & 1;
        // dV += P^T dO
        if (!mbar_wait(b_p_full, ph, ctl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t db = sStage(s) + C::ST_DO;
        const uint32_t qb = sStage(s) + C::ST_Q;
#pragma unroll
        for (int kk = 0; kk < C::BM / 16; ++kk)
          umma_ts(tmem + C::T_DV, tmem + C::T_S + kk * 8, sdesc_sw128(db + kk * 2048, C::QREG, 1024),
                  C::IDESC_KV, (it > 0) || (kk > 0));
        // next S^T
        const int s1 = (it + 1) % C::STAGES;
        if (it + 1 < n_iter) {
          if (!mbar_wait(b_qdo_full(s1), ((it + 1) / C::STAGES) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          issue_s(s1);
        }
        // dK += dS^T Q
        if (!mbar_wait(b_ds_full, ph, ctl)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BM / 16; ++kk)
          umma_ts(tmem + C::T_DK, tmem + C::T_DP + kk * 8, sdesc_sw128(qb + kk * 2048, C::QREG, 1024),
                  C::IDESC_KV, (it > 0) || (kk > 0));
        umma_commit(b_qdo_empty(s));
        // dQ^T = K^T dS^T
        const int buf = it & 1;
        if (it >= 2) {
          if (!mbar_wait(b_dq_free(buf), ((it >> 1) - 1) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          umma_ss(tmem + C::T_DQ + buf * C::BM, sdesc_sw128(sK + kk * 2048, C::KREG, 1024),
                  sdesc_sw128(sDS(buf) + kk * 2048, C::QREG, 1024), C::IDESC_Q, kk > 0);
        umma_commit(b_dq_full(buf));
        // next dP^T
        if (it + 1 < n_iter) issue_dp(s1);
      }
      if (ok) umma_commit(b_dkv_done);
      umma_commit(b_drain);
      mbar_wait_quiet(b_drain, 0, 200000000ull);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ P / dS warps (thread = key, 32 query columns)
    const int quarter = warp & 3;
    const int chalf = warp >> 2;                   // which 32 of the 64 query columns
    const int rloc = quarter * 32 + lane;
    const int key = k0 + rloc;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::T_S;
    const uint32_t tDP = tmem + lane_off + C::T_DP;
    const float c2 = args.scale_log2;
    const bool key_ok = key < args.N;
    const int col0 = 32 * chalf;
    bool ok = true;
    for (int it = 0; it < n_iter; ++it) {
      const int s = it % C::STAGES;
      const uint32_t ph = it & 1;
      const int q0 = (i_begin + it) * C::BM;
      const uint8_t* st = smem + C::OFF_ST + s * C::STAGE_STRIDE;
      const float* lse2 = reinterpret_cast<const float*>(st + C::ST_LSE) + col0;
      const float* dvec = reinterpret_cast<const float*>(st + C::ST_DV) + col0;
      if (!mbar_wait_warp(b_qdo_full(s), (it / C::STAGES) & 1, ctl)) { ok = false; break; }
      if (!mbar_wait_warp(b_s_full, ph, ctl)) { ok = false; break; }
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(tS + col0, r);
      tmem_wait_ld();
      reg_fence32(r);
      float p[32];
      // keys past the sequence end and (causal) queries before this key get P = 0
      const int cut = !key_ok ? C::BM : (args.causal ? key - q0 : 0);   // columns c < cut are masked
#pragma unroll
      for (int c = 0; c < 32; c += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c);
        const float2 x0 = ffma2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])),
                                make_float2(c2, c2), make_float2(-l4.x, -l4.y));
        const float2 x1 = ffma2(make_float2(__uint_as_float(r[c + 2]), __uint_as_float(r[c + 3])),
                                make_float2(c2, c2), make_float2(-l4.z, -l4.w));
        p[c + 0] = ex2_approx(x0.x);
        p[c + 1] = ex2_approx(x0.y);
        p[c + 2] = ex2_approx(x1.x);
        p[c + 3] = ex2_approx(x1.y);
      }
      if (cut > col0) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (col0 + c < cut) p[c] = 0.f;
      }
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(p[2 * c], p[2 * c + 1]);
      tmem_st16(tS + (col0 >> 1), pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(b_p_full);
      // dS = P (dP - D)
      if (!mbar_wait_warp(b_dp_full, ph, ctl)) { ok = false; break; }
      tc_fence_after();
      tmem_ld32(tDP + col0, r);
      tmem_wait_ld();
      reg_fence32(r);
#pragma unroll
      for (int c = 0; c < 32; c += 4) {
        const float4 d4 = *reinterpret_cast<const float4*>(dvec + c);
        const float2 a = fmul2(make_float2(p[c], p[c + 1]),
                               fsub2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), make_float2(d4.x, d4.y)));
        const float2 b = fmul2(make_float2(p[c + 2], p[c + 3]),
                               fsub2(make_float2(__uint_as_float(r[c + 2]), __uint_as_float(r[c + 3])), make_float2(d4.z, d4.w)));
        p[c] = a.x; p[c + 1] = a.y; p[c + 2] = b.x; p[c + 3] = b.y;
      }
#pragma unroll
      for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(p[2 * c], p[2 * c + 1]);
      tmem_st16(tDP + (col0 >> 1), pk);
      // this thread's half of the dS^T row into the swizzled smem buffer of this iteration
      const int buf = it & 1;
      if (it >= 2) {
        if (!mbar_wait_warp(b_dq_full(buf), ((it >> 1) - 1) & 1, ctl)) { ok = false; break; }
      }
      uint8_t* drow = smem + C::OFF_DS + buf * C::DS_BYTES + rloc * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int ch = 4 * chalf + q;
        const uint4 w = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        *reinterpret_cast<uint4*>(drow + ((ch ^ (rloc & 7)) << 4)) = w;
      }
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(b_ds_full);
    }
    // ---- epilogue: this thread's half of the dV, dK rows -> global
    if (ok && mbar_wait_warp(b_dkv_done, 0, ctl)) {
      tc_fence_after();
      const size_t grow = (static_cast<size_t>(bh) * args.N + key) * D + 64 * chalf;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t tsrc = tmem + lane_off + (which ? C::T_DK : C::T_DV) + 64 * chalf;
        __nv_bfloat16* dst = (which ? args.dk : args.dv) + grow;
        const float mul = which ? args.scale : 1.0f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
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
  } else if (warp < 12) {
    // ------------------------------------------------------------ dQ drain warpgroup (thread = head-dim lane)
    const int dl = (warp - 8) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp - 8) * 32) << 16;
    float* acc = args.dq_acc + static_cast<size_t>(bh) * args.N * D + dl;
    for (int it = 0; it < n_iter; ++it) {
      const int buf = it & 1;
      if (!mbar_wait_warp(b_dq_full(buf), (it >> 1) & 1, ctl)) break;
      tc_fence_after();
      uint32_t r[64];
      const uint32_t tq = tmem + lane_off + C::T_DQ + buf * C::BM;
      tmem_ld32(tq, *reinterpret_cast<uint32_t(*)[32]>(r));
      tmem_ld32(tq + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
      tmem_wait_ld();
      reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(r));
      reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(r + 32));
      tc_fence_before();
      mbar_arrive(b_dq_free(buf));
      const int q0 = (i_begin + it) * C::BM;
      const int nq = min(C::BM, args.N - q0);
      float* a_row = acc + static_cast<size_t>(q0) * D;
#pragma unroll
      for (int c = 0; c < 64; ++c)
        if (c < nq) red_add_f32(a_row + static_cast<size_t>(c) * D, __uint_as_float(r[c]));
    }
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
