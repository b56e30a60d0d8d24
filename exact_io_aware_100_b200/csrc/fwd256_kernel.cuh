// Forward attention kernel for head dim 256 (sm_100a).
//
// The nearauto.com FlashAttention-2 digest lists head dimensions up to 256
// among FlashAttention-2's additions ("新機能: 最大256のヘッドディメンション、マルチ
// クエリアテンション"); the computation is the same exact tiled attention with
// the online-softmax rescaling as for d = 64 / 128 (unite.ai page, "La
// Matematica dietro Flash Attention").  Sequences, lengths, strides and the
// bottom-right causal alignment follow layout.cuh.
//
// B200 layout of the work (tensor memory is the constraint: 128 lanes x 512
// columns of fp32 hold one 128 x 256 output accumulator and little else):
//  * persistent CTAs walk work tiles of 128 query rows of one (sequence, head);
//    causal tiles are visited longest first;
//  * blocks of 64 keys: S_j = Q K_j^T (M 128, N 64, K 256) into one of two
//    64-column score buffers, P_j (bf16) written back over it, and
//    O += P_j V_j (M 128, N 256, K 64) with A read from tensor memory;
//  * MMA issue order S_0, S_1, PV_0, S_2, PV_1, ...: the softmax of block j+1
//    runs while the tensor core computes P_j V_j and S_{j+2};
//  * TMA streams K_j, V_j (32 KB each) through a ring of five stages; Q
//    (64 KB) is loaded once per tile and released after the tile's last S;
//  * warps 0-3: softmax and epilogue (thread = query row = TMEM lane), warp 4
//    issues the MMAs from one thread, warp 5 issues the TMA loads;
//  * O is rescaled in tensor memory only when a row's block max exceeds its
//    reference max by more than 2^8 (exp2 units), after waiting for the
//    P V product that may still be adding into O;
//  * every mbarrier wait is bounded; on timeout the CTA sets the status word,
//    drains its own copies and MMAs, frees tensor memory and returns.
#pragma once

#include "fwd_kernel.cuh"
#include "layout.cuh"
#include "ptx.cuh"

namespace fa {

struct Fwd256Cfg {
  static constexpr int D = 256;
  static constexpr int BM = 128;                   // query rows per work tile
  static constexpr int BN = 64;                    // keys per block
  static constexpr int Q_REGION = 128 * 128;       // 64 columns (128 B) x 128 rows, bf16, 128-B swizzle
  static constexpr int KV_REGION = 64 * 128;       // 64 columns x 64 rows
  static constexpr int Q_BYTES = 4 * Q_REGION;     // 64 KB
  static constexpr int KV_BYTES = 4 * KV_REGION;   // 32 KB: one K or V tile of 64 keys
  static constexpr int STAGES = 5;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_S0 = 0, T_S1 = 64, T_O = 256;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = Q_BYTES;
  static constexpr int OFF_BAR = OFF_KV + STAGES * KV_BYTES;
  // barriers: q_full, q_empty, kv_full[S], kv_empty[S], s_full[2], p_full[2], pv_done, o_done, drain
  static constexpr int N_BARS = 2 + 2 * STAGES + 2 + 2 + 3;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;   // tmem slot, abort flag
  static constexpr int USED = OFF_MISC + 16;
  static constexpr int SMEM_BYTES = USED + 1024;          // + alignment slack
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, BN, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, false, true);
};
static_assert(Fwd256Cfg::SMEM_BYTES <= 232448, "shared memory plan");

// Key blocks (64 keys) tile qt (128 rows) of sequence s reads; 0 when the tile
// holds no query row or none of its rows sees a key.
__host__ __device__ __forceinline__ int fwd256_num_kv(const FwdArgs& a, const SeqSpan& s, int qt) {
  if (qt * 128 >= s.nq) return 0;
  const int n_all = (s.nk + 63) / 64;
  if (!a.causal) return n_all;
  const int last_row = min(qt * 128 + 127, s.nq - 1);
  const int vis = last_row + (s.nk - s.nq) + 1;       // keys < vis are visible to the last row
  return vis <= 0 ? 0 : min((vis + 63) / 64, n_all);
}

template <bool PACKED>
__global__ void __launch_bounds__(Fwd256Cfg::THREADS, 1)
fa_fwd256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const FwdArgs args) {
  using C = Fwd256Cfg;
  extern __shared__ __align__(16) uint8_t smem_raw[];   // only 16 B promised: the 1 KB rounding below is real
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  if (pad + C::USED > static_cast<uint32_t>(C::SMEM_BYTES)) {   // buffers do not fit: report, touch nothing
    if (threadIdx.x == 0) atomicOr(args.status, DEV_SMEM);
    return;
  }
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  const uint32_t sQ = sbase + C::OFF_Q;
  const uint32_t sKV = sbase + C::OFF_KV;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  const uint32_t b_q_full = bar0, b_q_empty = bar0 + 8;
  auto b_kv_full = [&](int s) { return bar0 + 16 + 8 * s; };
  auto b_kv_empty = [&](int s) { return bar0 + 16 + 8 * C::STAGES + 8 * s; };
  const uint32_t b_s_full0 = bar0 + 16 + 16 * C::STAGES;   // two: one per score buffer
  const uint32_t b_p_full0 = b_s_full0 + 16;               // two
  const uint32_t b_pv_done = b_p_full0 + 16;
  const uint32_t b_o_done = b_pv_done + 8;
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
    mbar_init(b_pv_done, 1);
    mbar_init(b_o_done, 1);
    mbar_init(b_drain, 1);
    fence_mbar_init();
  }
  if (warp == 4) tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
  if (warp == 5 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, args.status, args.wait_limit_ns};

  if (warp == 5) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t kv_it = 0, tile_cnt = 0;
      bool ok = true, q_pending = false;
      uint32_t q_parity = 0;
      uint32_t issued = 0, last_parity = 0;      // per-stage bit masks
      for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
        int b, h, qt;
        fwd_decode_tile(args, t, b, h, qt);
        const SeqSpan sp = seq_span<PACKED>(args.L, b, args.status);
        const int nkv = fwd256_num_kv(args, sp, qt);
        if (nkv == 0) continue;
        const int h_kv = h / args.group;
        if (tile_cnt > 0 && !mbar_wait(b_q_empty, (tile_cnt - 1) & 1, ctl)) { ok = false; break; }
        mbar_expect_tx(b_q_full, C::Q_BYTES);
        for (int r = 0; r < 4; ++r)
          tma_load_4d(sQ + r * C::Q_REGION, &tm_q, b_q_full, r * 64, sp.q0 + qt * 128, h, sp.bc);
        q_pending = true;
        q_parity = tile_cnt & 1;
        for (int j = 0; j < nkv && ok; ++j) {
          for (int kind = 0; kind < 2; ++kind, ++kv_it) {
            const int s = kv_it % C::STAGES;
            const uint32_t round = kv_it / C::STAGES;
            if (round > 0 && !mbar_wait(b_kv_empty(s), (round - 1) & 1, ctl)) { ok = false; break; }
            mbar_expect_tx(b_kv_full(s), C::KV_BYTES);
            const CUtensorMap* map = kind ? &tm_v : &tm_k;
            for (int r = 0; r < 4; ++r)
              tma_load_4d(sKV + s * C::KV_BYTES + r * C::KV_REGION, map, b_kv_full(s), r * 64, sp.k0 + j * 64, h_kv,
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
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop (its operands are warp-uniform) and one
    // elected lane issues each MMA and commit: measured faster than a loop run
    // by lane 0 alone.
    {
      constexpr uint32_t SBO = 1024;
      uint32_t kv_it = 0, tile_cnt = 0, g = 0;     // g: key blocks processed by this CTA, over all tiles
      bool ok = true;
      const uint64_t dq = sdesc_sw128(opaque_u32(sQ), 16, SBO);
      auto issue_s = [&](uint32_t d_tmem, uint32_t k_addr) {   // S = Q K^T, both K-major
        const uint64_t dk = sdesc_sw128(opaque_u32(k_addr), 16, SBO);
#pragma unroll
        for (int kk = 0; kk < C::D / 16; ++kk) {
          const uint32_t oa = ((kk >> 2) * C::Q_REGION + (kk & 3) * 32) >> 4;
          const uint32_t ob = ((kk >> 2) * C::KV_REGION + (kk & 3) * 32) >> 4;
          umma_ss_elect(d_tmem, dq + oa, dk + ob, C::IDESC_S, kk > 0);
        }
      };
      auto issue_pv = [&](uint32_t p_tmem, uint32_t v_addr, bool acc) {   // O += P V, V MN-major
        const uint64_t dv = sdesc_sw128(opaque_u32(v_addr), C::KV_REGION, SBO);
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          umma_ts_elect(tmem + C::T_O, p_tmem + kk * 8, dv + ((kk * 2048) >> 4), C::IDESC_PV, acc || (kk > 0));
      };
      // O += P_g V: wait for the softmax's P (buffer g & 1) and for V
      auto pv_step = [&](uint32_t gb, int sv, bool acc) -> bool {
        if (!mbar_wait_warp(b_p_full0 + 8 * (gb & 1), (gb >> 1) & 1, ctl)) return false;
        tc_fence_after();
        issue_pv(tmem + ((gb & 1) ? C::T_S1 : C::T_S0), sKV + sv * C::KV_BYTES, acc);
        umma_commit_elect(b_kv_empty(sv));
        umma_commit_elect(b_pv_done);
        return true;
      };
      for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
        int b, h, qt;
        fwd_decode_tile(args, t, b, h, qt);
        const int nkv = fwd256_num_kv(args, seq_span<PACKED>(args.L, b, args.status), qt);
        if (nkv == 0) continue;
        if (!mbar_wait_warp(b_q_full, tile_cnt & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        int sv_prev = 0;
        for (int j = 0; j < nkv; ++j, ++g) {
          // ---- S_j into buffer g & 1 (its previous P was read by PV_{g-2}, issued before)
          const int sk = kv_it % C::STAGES;
          if (!mbar_wait_warp(b_kv_full(sk), (kv_it / C::STAGES) & 1, ctl)) { ok = false; break; }
          ++kv_it;
          tc_fence_after();
          issue_s(tmem + ((g & 1) ? C::T_S1 : C::T_S0), sKV + sk * C::KV_BYTES);
          umma_commit_elect(b_s_full0 + 8 * (g & 1));
          umma_commit_elect(b_kv_empty(sk));
          if (j == nkv - 1) umma_commit_elect(b_q_empty);
          // ---- O += P_{j-1} V_{j-1}
          if (j > 0 && !pv_step(g - 1, sv_prev, j > 1)) { ok = false; break; }
          const int sv = kv_it % C::STAGES;
          if (!mbar_wait_warp(b_kv_full(sv), (kv_it / C::STAGES) & 1, ctl)) { ok = false; break; }
          ++kv_it;
          sv_prev = sv;
        }
        if (!ok) break;
        // ---- O += P_last V_last
        if (!pv_step(g - 1, sv_prev, nkv > 1)) { ok = false; break; }
        umma_commit_elect(b_o_done);
        ++tile_cnt;
      }
      // every MMA issued by this thread has completed before TMEM is freed
      umma_commit_elect(b_drain);
      mbar_wait_quiet(b_drain, 0, 200000000ull);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 0-3)
    const int rloc = warp * 32 + lane;                 // TMEM lane == row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tO = tmem + lane_off + C::T_O;
    const float c2 = args.scale_log2;
    uint32_t tile_cnt = 0, g = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < args.num_tiles && ok; t += gridDim.x) {
      int b, h, qt;
      fwd_decode_tile(args, t, b, h, qt);
      const SeqSpan sp = seq_span<PACKED>(args.L, b, args.status);
      const int nkv = fwd256_num_kv(args, sp, qt);
      const int row0 = qt * 128;                       // rows of the sequence
      const int row = row0 + rloc;
      if (nkv == 0) {                                  // no key visible to any row: O = 0, lse = -inf
        if (row < sp.nq) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.o) +
                                                row_offset(args.so, sp.bc, h, sp.q0 + row));
          for (int e = 0; e < C::D / 8; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
          args.lse[row_index<PACKED>(args.L, sp, h, row)] = -INFINITY;
        }
        continue;
      }
      const int off = sp.nk - sp.nq;                   // bottom-right causal alignment
      const int lim = args.causal ? min(row + off + 1, sp.nk) : sp.nk;        // keys < lim are visible
      const int lim_min = args.causal ? min(row0 + off + 1, sp.nk) : sp.nk;   // smallest lim in the tile
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < nkv; ++j, ++g) {
        const uint32_t tS = tmem + lane_off + ((g & 1) ? C::T_S1 : C::T_S0);
        if (!mbar_wait_warp(b_s_full0 + 8 * (g & 1), (g >> 1) & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(sr));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
        tmem_wait_ld();
        reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(sr));
        reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(sr + 32));
        float s[64];
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = __uint_as_float(sr[c]);
        const int kv0 = j * 64;
        if (kv0 + 64 > lim_min) {          // diagonal or tail block: mask keys >= lim
          const int cut = lim - kv0;
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= cut) s[c] = -INFINITY;
        }
        float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
        for (int c = 4; c < 60; c += 8) {
          mx0 = fmax3(mx0, s[c], s[c + 1]);
          mx1 = fmax3(mx1, s[c + 2], s[c + 3]);
          mx2 = fmax3(mx2, s[c + 4], s[c + 5]);
          mx3 = fmax3(mx3, s[c + 6], s[c + 7]);
        }
        mx0 = fmax3(mx0, s[60], s[61]);
        mx1 = fmax3(mx1, s[62], s[63]);
        const float mx = fmax3(mx0, mx1, fmaxf(mx2, mx3));
        const float m_new = fmaxf(m_ref, mx);
        const bool need = (m_new - m_ref) * c2 > 8.0f;          // false while the row has seen no key
        const bool rescale = __any_sync(0xffffffffu, need);   // warp-uniform decision
        float alpha = 1.0f;
        if (rescale) {
          alpha = m_new == -INFINITY ? 1.0f : ex2_approx((m_ref - m_new) * c2);
          l *= alpha;
          m_ref = m_new;
        }
        const float2 c2v = make_float2(c2, c2);
        const float m_use = m_ref == -INFINITY ? 0.0f : m_ref;
        const float2 negm = make_float2(-m_use * c2, -m_use * c2);
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
        uint32_t pr[32];
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
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
        tmem_st32(tS, pr);
        // O rescale: wait until P_{g-1} V (issued after S_g) has finished adding into O
        if (rescale && j > 0) {
          if (!mbar_wait_warp(b_pv_done, (g - 1) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
          for (int c = 0; c < C::D / 32; ++c) {
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
        mbar_arrive(b_p_full0 + 8 * (g & 1));
      }
      if (!ok) break;
      // ---- epilogue: O / l -> global, lse
      if (!mbar_wait_warp(b_o_done, tile_cnt & 1, ctl)) { ok = false; break; }
      tc_fence_after();
      const bool seen = m_ref != -INFINITY;            // a row that saw no key: O = 0, lse = -inf
      const float inv_l = seen ? 1.0f / l : 0.0f;
      const SeqSpan spe = seq_span<PACKED>(args.L, b, args.status);   // addresses formed after the loop
      const bool valid = row < spe.nq;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(args.o) + row_offset(args.so, spe.bc, h, spe.q0 + row);
#pragma unroll
      for (int c = 0; c < C::D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
        reg_fence32(o);
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
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
      if (valid)
        args.lse[row_index<PACKED>(args.L, spe, h, row)] =
            seen ? (m_ref * c2 + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      ++tile_cnt;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
