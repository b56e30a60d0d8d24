// Forward attention kernel for sm_100a: O = softmax(scale Q K^T) V, lse per row.
//
// The method (exact attention computed tile by tile with the online-softmax
// rescaling, so the N x N score matrix never leaves the chip) is the one the
// unite.ai page "Flash Attention: Rivoluzionando l'Efficienza dei Modelli
// Transformer" describes in "L'Algoritmo di Flash Attention" and "La Matematica
// dietro Flash Attention" (softmax decomposition and merge); the deferred
// normalisation and the skipping of fully masked causal tiles follow the
// nearauto.com FlashAttention-2 digest ("reducing non-matmul FLOPs", "better
// parallelism": query-row blocks spread over all SMs, sequence dimension too).
//
// B200 design (not the pages' A100 / H100 partitioning):
//  * persistent CTAs, one per SM, walk work tiles of 256 query rows of one
//    (sequence, head); causal tiles are visited longest first;
//  * any query and key lengths, fixed per batch entry or packed variable-length
//    sequences, and any row / head / batch strides (layout.cuh); TMA reads the
//    tiles through 4-D tensor maps [d][row][head][batch];
//  * warp roles: warps 0-3 and 4-7 are two softmax warpgroups, each owning one
//    128-row half of the tile (thread t owns TMEM lane / query row t); warp 8
//    issues the tcgen05 MMAs from one thread; warp 9 issues TMA loads from one
//    thread; warps 10-11 only take part in set-up and teardown;
//  * TMA streams K_j and V_j (128 keys each) through a ring of shared-memory
//    stages with full / empty mbarriers; Q (both halves) is loaded once per tile;
//  * tensor memory (512 columns): S0 | S1 | O0 | O1; P (bf16) is written back
//    over the first half of its S columns and fed to the P.V MMA from TMEM;
//  * MMA issue order per KV block j: S0_j, P1V_{j-1}, S1_j, P0V_j, so one
//    half's softmax overlaps the other half's MMAs (ping-pong);
//  * the softmax keeps a per-row reference max m and sum l; it rescales O in
//    TMEM only when the block max exceeds m by more than 2^8 in exp2 units
//    (exact: the final O / l uses the same reference), warp-uniformly;
//  * every mbarrier wait is bounded; on timeout the CTA sets the status word,
//    drains its own in-flight copies and MMAs, frees TMEM and returns.
#pragma once

#include "layout.cuh"
#include "ptx.cuh"

namespace fa {

struct FwdArgs {
  void* o;              // bf16 or f32, strides so
  float* lse;           // natural-log logsumexp, indexed by row_index
  uint32_t* status;     // device status word
  SeqLayout L;
  Strides so;           // element strides of o
  int group;            // query heads per key/value head (1: multi-head; H: multi-query)
  int n_qt;             // query tiles per sequence: ceil(L.Nq / tile rows)
  int num_tiles;        // B * H * n_qt
  int heads_per_group;  // causal tile order: heads whose K / V fit in L2 together
  int causal;
  int o_f32;
  float scale_log2;     // scale * log2(e)
  unsigned long long wait_limit_ns;
};

template <int D>
struct FwdCfg {
  static constexpr int BM = 128;                  // query rows per softmax warpgroup
  static constexpr int BN = 128;                  // keys per KV block
  static constexpr int TILE_M = 2 * BM;           // query rows per work tile
  static constexpr int REGION = 128 * 128;        // one 64-column (128 B) swizzle region of a 128-row tile
  static constexpr int N_REG = D / 64;            // regions per 128-row tile
  static constexpr int Q_HALF = BM * D * 2;       // bytes of one 128-row Q half
  static constexpr int KV_BYTES = BN * D * 2;     // bytes of one K or V block
  static constexpr int STAGES = (D == 128) ? 4 : 8;
  static constexpr int THREADS = 384;
  // Register split (setmaxnreg): 384 threads launch with 168 registers each
  // (three warps per sub-partition); the eight softmax warps take 224, the
  // other four give theirs down to 56: 256 * 224 + 128 * 56 = 384 * 168.  It
  // also balances within each sub-partition, where setmaxnreg.inc draws its
  // registers from: two softmax warps take 2 * (224 - 168) = 112, which the one
  // other warp there frees (168 - 56).
  static constexpr int LAUNCH_REGS = 168;
  static_assert(2 * (224 - LAUNCH_REGS) <= LAUNCH_REGS - 56,
                "register split does not balance within a sub-partition");
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S0 = 0, T_S1 = 128, T_O0 = 256, T_O1 = 256 + D;
  // shared-memory layout (offsets from a 1024-aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * Q_HALF;
  static constexpr int OFF_BAR = OFF_KV + STAGES * KV_BYTES;
  // barriers: q_full, q_empty, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_done, drain
  static constexpr int N_BARS = 2 + 2 * STAGES + 2 + 2 + 2;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;   // tmem slot, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024; // + alignment slack
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, false, true);
};

// Work tile t -> (sequence b, query head h, tile qt of query rows).  Query
// head h reads key/value head h / group (sets of consecutive query heads share
// one: grouped-query attention; group = 1 is multi-head).
__host__ __device__ __forceinline__ void fwd_decode_tile(const FwdArgs& a, int t, int& b, int& h, int& qt) {
  const int bh_all = a.L.B * a.L.H;
  int bh;
  if (a.causal) {            // heads in groups whose K / V fit in L2 together; longest work first in a group
    const int per_group = a.heads_per_group * a.n_qt;
    const int g = t / per_group;
    const int r = t - g * per_group;
    const int h0 = g * a.heads_per_group;
    const int gh = min(a.heads_per_group, bh_all - h0);
    qt = a.n_qt - 1 - r / gh;
    bh = h0 + r % gh;
  } else {                   // neighbouring CTAs share a head's K / V in L2
    bh = t / a.n_qt;
    qt = t % a.n_qt;
  }
  b = bh / a.L.H;
  h = bh - b * a.L.H;
}

// Key blocks (128 keys) tile qt of sequence s reads; 0 when the tile holds no
// query row or none of its rows sees a key (then its rows are written as empty).
__host__ __device__ __forceinline__ int fwd_num_kv(const FwdArgs& a, const SeqSpan& s, int qt) {
  if (qt * 256 >= s.nq) return 0;
  const int n_all = (s.nk + 127) / 128;
  if (!a.causal) return n_all;
  const int last_row = min(qt * 256 + 255, s.nq - 1);
  const int vis = last_row + (s.nk - s.nq) + 1;       // keys < vis are visible to the last row
  return vis <= 0 ? 0 : min((vis + 127) / 128, n_all);
}

template <int D, bool PACKED>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const FwdArgs args) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sKV = sbase + C::OFF_KV;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t b_q_full = bar0, b_q_empty = bar0 + 8;
  auto b_kv_full = [&](int s) { return bar0 + 16 + 8 * s; };
  auto b_kv_empty = [&](int s) { return bar0 + 16 + 8 * C::STAGES + 8 * s; };
  const uint32_t b_s_full0 = bar0 + 16 + 16 * C::STAGES;
  const uint32_t b_p_full0 = b_s_full0 + 16;
  const uint32_t b_o_done = b_p_full0 + 16;
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
    mbar_init(b_s_full0, 1);
    mbar_init(b_s_full0 + 8, 1);
    mbar_init(b_p_full0, 128);
    mbar_init(b_p_full0 + 8, 128);
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
        const int nkv = fwd_num_kv(args, sp, qt);
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
              tma_load_4d(sKV + s * C::KV_BYTES + r * C::REGION, map, b_kv_full(s), r * 64, sp.k0 + j * 128, h_kv,
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
      constexpr uint32_t LBO_K = 16, LBO_V = C::REGION, SBO = 1024;
      uint32_t kv_it = 0, tile_cnt = 0, p_par0 = 0, p_par1 = 0;
      bool ok = true;
      auto issue_s = [&](uint32_t d_tmem, uint32_t q_addr, uint32_t k_addr) {   // S = Q K^T
        const uint64_t dq = sdesc_sw128(opaque_u32(q_addr), LBO_K, SBO);
        const uint64_t dk = sdesc_sw128(opaque_u32(k_addr), LBO_K, SBO);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * C::REGION + (kk & 3) * 32) >> 4;
          umma_ss_elect(d_tmem, dq + off, dk + off, C::IDESC_S, kk > 0);
        }
      };
      auto issue_pv = [&](uint32_t d_tmem, uint32_t p_tmem, uint32_t v_addr, bool acc) {   // O += P V
        const uint64_t dv = sdesc_sw128(opaque_u32(v_addr), LBO_V, SBO);
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          umma_ts_elect(d_tmem, p_tmem + kk * 8, dv + ((kk * 2048) >> 4), C::IDESC_PV, acc || (kk > 0));
      };
      for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
        int b, h, qt;
        fwd_decode_tile(args, t, b, h, qt);
        const int nkv = fwd_num_kv(args, seq_span<PACKED>(args.L, b, args.status), qt);
        if (nkv == 0) continue;
        if (!mbar_wait_warp(b_q_full, tile_cnt & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        int sv_prev = 0;
        for (int j = 0; j < nkv; ++j) {
          // ---- K_j: S0 = Q0 K^T
          const int sk = kv_it % C::STAGES;
          if (!mbar_wait_warp(b_kv_full(sk), (kv_it / C::STAGES) & 1, ctl)) { ok = false; break; }
          ++kv_it;
          tc_fence_after();
          const uint32_t kbase = sKV + sk * C::KV_BYTES;
          issue_s(tmem + C::T_S0, sQ, kbase);
          umma_commit_elect(b_s_full0);
          // ---- O1 += P1 V_{j-1}
          if (j > 0) {
            if (!mbar_wait_warp(b_p_full0 + 8, p_par1, ctl)) { ok = false; break; }
            p_par1 ^= 1;
            tc_fence_after();
            issue_pv(tmem + C::T_O1, tmem + C::T_S1, sKV + sv_prev * C::KV_BYTES, j > 1);
            umma_commit_elect(b_kv_empty(sv_prev));
          }
          // ---- S1 = Q1 K^T
          issue_s(tmem + C::T_S1, sQ + C::Q_HALF, kbase);
          umma_commit_elect(b_s_full0 + 8);
          umma_commit_elect(b_kv_empty(sk));
          if (j == nkv - 1) umma_commit_elect(b_q_empty);
          // ---- V_j: O0 += P0 V_j
          const int sv = kv_it % C::STAGES;
          if (!mbar_wait_warp(b_kv_full(sv), (kv_it / C::STAGES) & 1, ctl)) { ok = false; break; }
          ++kv_it;
          if (!mbar_wait_warp(b_p_full0, p_par0, ctl)) { ok = false; break; }
          p_par0 ^= 1;
          tc_fence_after();
          issue_pv(tmem + C::T_O0, tmem + C::T_S0, sKV + sv * C::KV_BYTES, j > 0);
          sv_prev = sv;
        }
        if (!ok) break;
        // ---- O1 += P1 V_last
        if (!mbar_wait_warp(b_p_full0 + 8, p_par1, ctl)) { ok = false; break; }
        p_par1 ^= 1;
        tc_fence_after();
        issue_pv(tmem + C::T_O1, tmem + C::T_S1, sKV + sv_prev * C::KV_BYTES, nkv > 1);
        umma_commit_elect(b_kv_empty(sv_prev));
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
    const uint32_t b_s_full = b_s_full0 + 8 * half;
    const uint32_t b_p_full = b_p_full0 + 8 * half;
    const float c2 = args.scale_log2;
    uint32_t s_par = 0, tile_cnt = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
      int b, h, qt;
      fwd_decode_tile(args, t, b, h, qt);
      const SeqSpan sp = seq_span<PACKED>(args.L, b, args.status);
      const int nkv = fwd_num_kv(args, sp, qt);
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
        uint32_t sr[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sr + c * 32));
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(sr + c * 32));
        float s[128];
#pragma unroll
        for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
        const int kv0 = j * 128;
        if (kv0 + 128 > lim_min) {          // diagonal or tail block: mask keys >= lim
          const int cut = lim - kv0;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= cut) s[c] = -INFINITY;
        }
        // row max: four independent chains of 3-input max
        float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
        for (int c = 4; c < 124; c += 8) {
          mx0 = fmax3(mx0, s[c], s[c + 1]);
          mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
          mx2 = fmax3(mx2, s[c + 4], s[c + 5]);
          mx3 = fmax3(mx3, s[c + 6], s[c + 7]);
        }
        mx0 = fmax3(mx0, s[124], s[125]);
        mx1 = fmax3(mx1, s[126], s[127]);
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
        uint32_t pr[64];
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
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
        tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(pr));
        tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(pr + 32));
        // O rescale (after the scores are dead, to keep register pressure down).
        // Safe: S_j's commit covered every earlier MMA, including P V_{j-1} into O.
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
