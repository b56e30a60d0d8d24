// Forward attention kernel for sm_100a at head dim 64.
//
// Same method, tiling, scheduler and layouts as fwd_kernel.cuh (exact
// attention tile by tile with the online-softmax rescaling: the unite.ai page
// "Flash Attention: Rivoluzionando l'Efficienza dei Modelli Transformer",
// "L'Algoritmo di Flash Attention" and "La Matematica dietro Flash Attention";
// the nearauto.com FlashAttention-2 digest for the deferred normalisation and
// the skipped causal tiles), with the order of the products changed for the
// shape: at d = 64 a 128 x 128 score block costs half the tensor time of
// d = 128 while its softmax costs the same, so waiting for the next block's
// scores must leave the softmax path.
//
//  * tensor memory (512 columns): S0 | S1 | O0 | O1 | P0 | P1 (128, 128, 64,
//    64, 64, 64); P has columns of its own instead of overwriting S;
//  * as soon as a softmax warpgroup has read S_j into registers it releases
//    the S buffer (s_free) and the MMA warp computes S_{j+1} into it while the
//    softmax still works on block j; the products run in the order
//    S0_{j+1}, S1_{j+1}, P0 V_j, P1 V_j, so each half finds its next scores
//    ready when it finishes a block;
//  * P_j is written after P_{j-1} V has completed (pv_done), and O is rescaled
//    only after that as well;
//  * warp roles, the K / V ring, the persistent tile walk, the lazy rescale
//    (only when the block max exceeds the reference by more than 2^8 in exp2
//    units), the epilogue and the bounded waits are those of fwd_kernel.cuh.
#pragma once

#include "fwd_kernel.cuh"

namespace fa {

template <int D_, int BN_>
struct FwdSpCfg {
  static constexpr int D = D_;
  static constexpr int BM = 128;                  // query rows per softmax warpgroup
  static constexpr int BN = BN_;                  // keys per KV block
  static constexpr int REGION = 128 * 128;        // one 64-column (128 B) swizzle region of a 128-row Q half
  static constexpr int KV_REGION = BN * 128;      // one 64-column region of a BN-row K or V block
  static constexpr int N_REG = D / 64;            // regions per row
  static constexpr int Q_HALF = BM * D * 2;       // bytes of one 128-row Q half
  static constexpr int KV_BYTES = BN * D * 2;     // bytes of one K or V block
  static constexpr int STAGES = 8;
  static constexpr int THREADS = 384;
  // Register split as in fwd_kernel.cuh: 384 threads launch with 168 registers;
  // the eight softmax warps take 224, the other four give theirs down to 56.
  static constexpr int LAUNCH_REGS = 168;
  static_assert(2 * (224 - LAUNCH_REGS) <= LAUNCH_REGS - 56,
                "register split does not balance within a sub-partition");
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_O0 = 0, T_O1 = D, T_S0 = 2 * D, T_S1 = 2 * D + BN, T_P0 = 2 * D + 2 * BN,
                            T_P1 = 2 * D + 2 * BN + BN / 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * Q_HALF;
  static constexpr int OFF_BAR = OFF_KV + STAGES * KV_BYTES;
  // barriers: q_full, q_empty, kv_full[S], kv_empty[S], s_full[2], s_free[2], p_full[2], pv_done[2], o_done, drain
  static constexpr int N_BARS = 2 + 2 * STAGES + 8 + 2;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;   // tmem slot, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024; // + alignment slack
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, false, true);
  static_assert(T_P1 + BN / 2 <= TMEM_COLS, "tensor memory plan");
  static_assert(SMEM_BYTES <= 232448, "shared memory plan");
};
using Fwd64Cfg = FwdSpCfg<64, 128>;

// Key blocks of BN keys that tile qt (256 query rows) of sequence s reads.
template <int BN>
__host__ __device__ __forceinline__ int fwd_num_kv_bn(const FwdArgs& a, const SeqSpan& s, int qt) {
  if (qt * 256 >= s.nq) return 0;
  const int n_all = (s.nk + BN - 1) / BN;
  if (!a.causal) return n_all;
  const int last_row = min(qt * 256 + 255, s.nq - 1);
  const int vis = last_row + (s.nk - s.nq) + 1;       // keys < vis are visible to the last row
  return vis <= 0 ? 0 : min((vis + BN - 1) / BN, n_all);
}

template <int D_, int BN_, bool PACKED>
__global__ void __launch_bounds__(FwdSpCfg<D_, BN_>::THREADS, 1)
fa_fwd_sp_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const FwdArgs args) {
  using C = FwdSpCfg<D_, BN_>;
  constexpr int D = C::D, BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sKV = sbase + C::OFF_KV;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t b_q_full = bar0, b_q_empty = bar0 + 8;
  auto b_kv_full = [&](int s) { return bar0 + 16 + 8 * s; };
  auto b_kv_empty = [&](int s) { return bar0 + 16 + 8 * C::STAGES + 8 * s; };
  const uint32_t b_s_full0 = bar0 + 16 + 16 * C::STAGES;   // [half]: S_j in the half's S buffer
  const uint32_t b_s_free0 = b_s_full0 + 16;                // [half]: the softmax has read S_j
  const uint32_t b_p_full0 = b_s_free0 + 16;                // [half]: P_j in the half's P buffer
  const uint32_t b_pv_done0 = b_p_full0 + 16;               // [half]: P_j V_j has completed
  const uint32_t b_o_done = b_pv_done0 + 16;
  const uint32_t b_drain = b_o_done + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *abort_flag = 0u;
    mbar_init(b_q_full, 1);
    mbar_init(b_q_empty, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(b_kv_full(s), 1);
      mbar_init(b_kv_empty(s), 1);
    }
    for (int hf = 0; hf < 2; ++hf) {
      mbar_init(b_s_full0 + 8 * hf, 1);
      mbar_init(b_s_free0 + 8 * hf, 128);
      mbar_init(b_p_full0 + 8 * hf, 128);
      mbar_init(b_pv_done0 + 8 * hf, 1);
    }
    mbar_init(b_o_done, 1);
    mbar_init(b_drain, 1);
    fence_mbar_init();
  }
  if (warp == 8) tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
  if (warp == 9 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, args.status, args.wait_limit_ns};
  // Register split, taken inside each role's branch so the compiler sees which
  // budget governs which code: 384 threads x 168 registers at launch
  // = 128 x (224 + 224) for the softmax warpgroups + 128 x 56 for warps 8-11.
  if (warp == 9) {
    // ------------------------------------------------------------ TMA producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;");
    if (lane == 0) {
      uint32_t kv_it = 0, tile_cnt = 0;
      bool ok = true, q_pending = false;
      uint32_t q_parity = 0;
      uint32_t issued = 0, last_parity = 0;      // per-stage bit masks
      for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
        int b, h, qt;
        fwd_decode_tile(args, t, b, h, qt);
        const SeqSpan sp = seq_span<PACKED>(args.L, b, args.status);
        const int nkv = fwd_num_kv_bn<BN>(args, sp, qt);
        if (nkv == 0) continue;                        // nothing to load for this tile
        const int h_kv = h / args.group;
        if (tile_cnt > 0 && !mbar_wait(b_q_empty, (tile_cnt - 1) & 1, ctl)) { ok = false; break; }
        mbar_expect_tx(b_q_full, 2 * C::Q_HALF);
        for (int hf = 0; hf < 2; ++hf)
          for (int r = 0; r < C::N_REG; ++r)
            tma_load_4d(sQ + hf * C::Q_HALF + r * C::REGION, &tm_q, b_q_full, r * 64, sp.q0 + qt * 256 + hf * 128,
                        h, sp.bc);
        q_pending = true;
        q_parity = tile_cnt & 1;
        for (int j = 0; j < nkv && ok; ++j) {
          for (int kind = 0; kind < 2; ++kind, ++kv_it) {
            const int s = kv_it % C::STAGES;
            const uint32_t round = kv_it / C::STAGES;
            if (round > 0 && !mbar_wait(b_kv_empty(s), (round - 1) & 1, ctl)) { ok = false; break; }
            mbar_expect_tx(b_kv_full(s), C::KV_BYTES);
            const CUtensorMap* map = kind ? &tm_v : &tm_k;
            for (int r = 0; r < C::N_REG; ++r)
              tma_load_4d(sKV + s * C::KV_BYTES + r * C::KV_REGION, map, b_kv_full(s), r * 64, sp.k0 + j * BN, h_kv,
                          sp.bc);
            issued |= 1u << s;
            last_parity = (last_parity & ~(1u << s)) | ((round & 1u) << s);
          }
        }
        ++tile_cnt;
      }
      if (!ok) {   // drain our own copies still in flight before the CTA exits
        for (int s = 0; s < C::STAGES; ++s)
          if ((issued >> s) & 1u) mbar_wait_quiet(b_kv_full(s), (last_parity >> s) & 1u, 200000000ull);
        if (q_pending) mbar_wait_quiet(b_q_full, q_parity, 200000000ull);
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop (its operands are warp-uniform) and one
    // elected lane issues each MMA and commit: measured faster than a loop run
    // by lane 0 alone.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;");
    {
      // descriptor of address a + off == descriptor of a, plus off / 16 (no carry:
      // shared addresses stay below 2^18, the start field holds 14 bits of a / 16)
      constexpr uint32_t LBO_K = 16, LBO_V = C::KV_REGION, SBO = 1024;
      uint32_t kv_it = 0, tile_cnt = 0;
      bool ok = true;
      auto issue_s = [&](uint32_t d_tmem, uint32_t q_addr, uint32_t k_addr) {   // S = Q K^T
        const uint64_t dq = sdesc_sw128(opaque_u32(q_addr), LBO_K, SBO);
        const uint64_t dk = sdesc_sw128(opaque_u32(k_addr), LBO_K, SBO);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offq = ((kk >> 2) * C::REGION + (kk & 3) * 32) >> 4;
          const uint32_t offk = ((kk >> 2) * C::KV_REGION + (kk & 3) * 32) >> 4;
          umma_ss_elect(d_tmem, dq + offq, dk + offk, C::IDESC_S, kk > 0);
        }
      };
      auto issue_pv = [&](uint32_t d_tmem, uint32_t p_tmem, uint32_t v_addr, bool acc) {   // O += P V
        const uint64_t dv = sdesc_sw128(opaque_u32(v_addr), LBO_V, SBO);
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          umma_ts_elect(d_tmem, p_tmem + kk * 8, dv + ((kk * 2048) >> 4), C::IDESC_PV, acc || (kk > 0));
      };
      // K_j and V_j are the ring's loads 2j and 2j + 1 of a tile (kv_base + ...)
      auto stage_of = [&](uint32_t n) { return static_cast<int>(n % C::STAGES); };
      auto parity_of = [&](uint32_t n) { return (n / C::STAGES) & 1u; };
      uint32_t s_par[2] = {0u, 0u}, p_par[2] = {0u, 0u};
      for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
        int b, h, qt;
        fwd_decode_tile(args, t, b, h, qt);
        const int nkv = fwd_num_kv_bn<BN>(args, seq_span<PACKED>(args.L, b, args.status), qt);
        if (nkv == 0) continue;
        const uint32_t kv_base = kv_it;
        kv_it += 2u * static_cast<uint32_t>(nkv);
        if (!mbar_wait_warp(b_q_full, tile_cnt & 1, ctl)) { ok = false; break; }
        // ---- prologue: S0_0, S1_0 (the S buffers were released by the previous tile's last reads)
        {
          const uint32_t nk = kv_base;
          if (!mbar_wait_warp(b_kv_full(stage_of(nk)), parity_of(nk), ctl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kbase = sKV + stage_of(nk) * C::KV_BYTES;
          for (int hf = 0; hf < 2; ++hf) {
            if (tile_cnt > 0) {
              if (!mbar_wait_warp(b_s_free0 + 8 * hf, s_par[hf], ctl)) { ok = false; break; }
              s_par[hf] ^= 1u;
              tc_fence_after();
            }
            issue_s(tmem + (hf ? C::T_S1 : C::T_S0), sQ + hf * C::Q_HALF, kbase);
            umma_commit_elect(b_s_full0 + 8 * hf);
          }
          if (!ok) break;
          umma_commit_elect(b_kv_empty(stage_of(nk)));
        }
        for (int j = 0; j < nkv; ++j) {
          // ---- S_{j+1} of both halves, each as soon as its softmax has read S_j
          if (j + 1 < nkv) {
            const uint32_t nk = kv_base + 2u * (j + 1);
            if (!mbar_wait_warp(b_kv_full(stage_of(nk)), parity_of(nk), ctl)) { ok = false; break; }
            const uint32_t kbase = sKV + stage_of(nk) * C::KV_BYTES;
            for (int hf = 0; hf < 2; ++hf) {
              if (!mbar_wait_warp(b_s_free0 + 8 * hf, s_par[hf], ctl)) { ok = false; break; }
              s_par[hf] ^= 1u;
              tc_fence_after();
              issue_s(tmem + (hf ? C::T_S1 : C::T_S0), sQ + hf * C::Q_HALF, kbase);
              umma_commit_elect(b_s_full0 + 8 * hf);
            }
            if (!ok) break;
            umma_commit_elect(b_kv_empty(stage_of(nk)));
          }
          // ---- O_h += P_h V_j, each as soon as its softmax has written P_j
          const uint32_t nv = kv_base + 2u * j + 1u;
          if (!mbar_wait_warp(b_kv_full(stage_of(nv)), parity_of(nv), ctl)) { ok = false; break; }
          const uint32_t vbase = sKV + stage_of(nv) * C::KV_BYTES;
          for (int hf = 0; hf < 2; ++hf) {
            if (!mbar_wait_warp(b_p_full0 + 8 * hf, p_par[hf], ctl)) { ok = false; break; }
            p_par[hf] ^= 1u;
            tc_fence_after();
            issue_pv(tmem + (hf ? C::T_O1 : C::T_O0), tmem + (hf ? C::T_P1 : C::T_P0), vbase, j > 0);
            umma_commit_elect(b_pv_done0 + 8 * hf);
          }
          if (!ok) break;
          umma_commit_elect(b_kv_empty(stage_of(nv)));
        }
        if (!ok) break;
        umma_commit_elect(b_q_empty);
        umma_commit_elect(b_o_done);
        ++tile_cnt;
      }
      // every MMA issued by this thread has completed before TMEM is freed
      umma_commit_elect(b_drain);
      mbar_wait_quiet(b_drain, 0, 200000000ull);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax warpgroups
    asm volatile("setmaxnreg.inc.sync.aligned.u32 224;");
    const int half = warp >> 2;                       // which 128-row half
    const int rloc = (warp & 3) * 32 + lane;          // TMEM lane == row within the half
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + (half ? C::T_S1 : C::T_S0);
    const uint32_t tO = tmem + lane_off + (half ? C::T_O1 : C::T_O0);
    const uint32_t tP = tmem + lane_off + (half ? C::T_P1 : C::T_P0);
    const uint32_t b_s_full = b_s_full0 + 8 * half;
    const uint32_t b_s_free = b_s_free0 + 8 * half;
    const uint32_t b_p_full = b_p_full0 + 8 * half;
    const uint32_t b_pv_done = b_pv_done0 + 8 * half;
    const float c2 = args.scale_log2;
    uint32_t s_par = 0, tile_cnt = 0;
    uint32_t blocks = 0;                              // blocks this half has processed (all tiles)
    bool ok = true;
    for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
      int b, h, qt;
      fwd_decode_tile(args, t, b, h, qt);
      const SeqSpan sp = seq_span<PACKED>(args.L, b, args.status);
      const int nkv = fwd_num_kv_bn<BN>(args, sp, qt);
      const int row0 = qt * 256 + half * 128;           // rows of the sequence
      const int row = row0 + rloc;
      if (nkv == 0) {                                   // no key visible to any row: O = 0, lse = -inf
        if (row < sp.nq) {
          const long long o_off = row_offset(args.so, sp.bc, h, sp.q0 + row);
          const long long l_idx = row_index<PACKED>(args.L, sp, h, row);
          if (args.o_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(args.o) + o_off);
            for (int e = 0; e < D / 4; ++e) dst[e] = make_float4(0.f, 0.f, 0.f, 0.f);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.o) + o_off);
            for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
          }
          args.lse[l_idx] = -INFINITY;
        }
        continue;
      }
      const int off = sp.nk - sp.nq;                    // bottom-right causal alignment
      const int lim = args.causal ? min(row + off + 1, sp.nk) : sp.nk;        // keys < lim are visible
      const int lim_min = args.causal ? min(row0 + off + 1, sp.nk) : sp.nk;   // smallest lim in the warpgroup
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < nkv; ++j) {
        if (!mbar_wait_warp(b_s_full, s_par, ctl)) { ok = false; break; }
        s_par ^= 1;
        tc_fence_after();
        uint32_t sr[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c)
          tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sr + c * 32));
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(sr + c * 32));
        tc_fence_before();
        mbar_arrive(b_s_free);                          // the MMA warp may compute S_{j+1} into the buffer
        float s[BN];
#pragma unroll
        for (int c = 0; c < BN; ++c) s[c] = __uint_as_float(sr[c]);
        const int kv0 = j * BN;
        if (kv0 + BN > lim_min) {           // diagonal or tail block: mask keys >= lim
          const int cut = lim - kv0;
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c >= cut) s[c] = -INFINITY;
        }
        // row max: four independent chains of 3-input max
        float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
        for (int c = 4; c < BN - 4; c += 8) {
          mx0 = fmax3(mx0, s[c], s[c + 1]);
          mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
          mx2 = fmax3(mx2, s[c + 4], s[c + 5]);
          mx3 = fmax3(mx3, s[c + 6], s[c + 7]);
        }
        mx0 = fmax3(mx0, s[BN - 4], s[BN - 3]);
        mx1 = fmax3(mx1, s[BN - 2], s[BN - 1]);
        const float mx = fmax3(mx0, mx1, fmaxf(mx2, mx3));
        const float m_new = fmaxf(m_ref, mx);
        const bool need = (m_new - m_ref) * c2 > 8.0f;          // false while the row has seen no key
        const bool rescale = __any_sync(0xffffffffu, need);   // warp-uniform decision
        float alpha = 1.0f;
        if (rescale) {
          // 0 on a row's first visible key (m_ref = -inf); 1 while it has seen none
          alpha = m_new == -INFINITY ? 1.0f : ex2_approx((m_ref - m_new) * c2);
          l *= alpha;
          m_ref = m_new;
        }
        // p = 2^(s c2 - m c2): three of every eight pairs on the FMA pipe, the rest
        // on the special-function unit.  A row that has seen no key yet has only
        // masked scores here, and a finite reference keeps them at (about) zero.
        const float2 c2v = make_float2(c2, c2);
        const float m_use = m_ref == -INFINITY ? 0.0f : m_ref;
        const float2 negm = make_float2(-m_use * c2, -m_use * c2);
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
        uint32_t pr[BN / 2];
#pragma unroll
        for (int c = 0; c < BN; c += 2) {
          const float2 x = ffma2(make_float2(s[c], s[c + 1]), c2v, negm);
          float2 p;
          if ((0x92u >> ((c >> 1) & 7)) & 1u) {
            p = ex2_poly2(x);
          } else {
            p.x = ex2_approx(x.x);
            p.y = ex2_approx(x.y);
          }
          if ((c >> 1) & 1) acc1 = fadd2(acc1, p); else acc0 = fadd2(acc0, p);
          pr[c >> 1] = pack_bf16x2(p.x, p.y);
        }
        const float2 acc = fadd2(acc0, acc1);
        l += acc.x + acc.y;
        // P_{j-1} V (the previous block's, possibly of the previous tile) must have
        // read the P buffer and added into O before P_j overwrites it or O is rescaled
        if (blocks > 0 && !mbar_wait_warp(b_pv_done, (blocks - 1) & 1, ctl)) { ok = false; break; }
        ++blocks;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) tmem_st32(tP + c * 32, *reinterpret_cast<uint32_t(*)[32]>(pr + c * 32));
        // O rescale (after the scores are dead, to keep register pressure down)
        if (rescale && j > 0) {
          const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
            reg_fence32(o);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float2 v = fmul2(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2);
              o[e] = __float_as_uint(v.x);
              o[e + 1] = __float_as_uint(v.y);
            }
            tmem_st32(tO + c * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(b_p_full);
      }
      if (!ok) break;
      // ---- epilogue: O / l -> global, lse
      if (!mbar_wait_warp(b_o_done, tile_cnt & 1, ctl)) { ok = false; break; }
      tc_fence_after();
      // a row that saw no key (m_ref still -inf) is written as O = 0, lse = -inf
      const bool seen = m_ref != -INFINITY;
      const float inv_l = seen ? 1.0f / l : 0.0f;
      const SeqSpan spe = seq_span<PACKED>(args.L, b, args.status);   // addresses formed after the loop
      const bool valid = row < spe.nq;
      const long long o_off = row_offset(args.so, spe.bc, h, spe.q0 + row);
      const long long l_idx = row_index<PACKED>(args.L, spe, h, row);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
        reg_fence32(o);
        if (valid) {
          if (args.o_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(args.o) + o_off + c * 32);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv_l, __uint_as_float(o[4 * e + 1]) * inv_l,
                                   __uint_as_float(o[4 * e + 2]) * inv_l, __uint_as_float(o[4 * e + 3]) * inv_l);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.o) + o_off + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(o[8 * e + 0]) * inv_l, __uint_as_float(o[8 * e + 1]) * inv_l);
              w.y = pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv_l, __uint_as_float(o[8 * e + 3]) * inv_l);
              w.z = pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv_l, __uint_as_float(o[8 * e + 5]) * inv_l);
              w.w = pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv_l, __uint_as_float(o[8 * e + 7]) * inv_l);
              dst[e] = w;
            }
          }
        }
      }
      if (valid) args.lse[l_idx] = seen ? (m_ref * c2 + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      ++tile_cnt;
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 56;");   // warps 10-11: set-up and teardown only
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
