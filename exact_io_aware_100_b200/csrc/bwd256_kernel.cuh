// Backward attention kernel for sm_100a at head dim 256.
//
// Same method and formulas as bwd_kernel.cuh (the deepfa.ir page "Flash
// Attention: بهینه‌سازی مکانیزم توجه در ترنسفورمرها", section "تکنیک 2: محاسبه
// مجدد": P is recomputed from Q, K and the saved logsumexp; the nearauto.com
// FlashAttention-2 digest, "better parallelism": each worker owns a block of
// keys), at the head dimension the digest's section "新機能: 最大256のヘッド
// ディメンション、マルチクエリアテンション" adds.
//
// Why a kernel of its own: the fp32 dK and dV of 128 keys at d = 256 alone fill
// the 512 tensor-memory columns of an SM.  So each 128-key block is handled by
// two CTAs, CTA c owning columns [128 c, 128 c + 128) of d:
//   S^T  = K Q^T        (full d, computed by both CTAs)       TMEM S
//   dP^T = V dO^T       (full d, computed by both CTAs)       TMEM DP
//   dV_c += P^T dO_c    (A = P^T bf16 in TMEM)                TMEM DV
//   dK_c += dS^T Q_c    (A = dS^T bf16, shared memory)        TMEM DK
//   dQ^T_c = K_c^T dS^T (into TMEM DQ, added to dQacc by tensor bulk reductions)
// per block of 64 queries (K, V: 64 KB each, resident; a 64-query block of Q
// or dO is 32 KB).  Tensor memory: DV 128 | DK 128 | S 64 | DP 64 | DQ 64 |
// P 32 (of 512) columns.  Q and dO are staged as two 16 KB halves of d each:
// the half the CTA does not own is read only by S^T (dP^T) and is reloaded for
// the next block as soon as that product completes; the owned half is kept
// until dK (dV) has read it.  The MMA thread issues the next block's S^T over
// the early half first, so the owned half's load overlaps dQ^T and that half.
//
// Warp roles (448 threads): warps 0-7 compute P and dS (thread = key row,
// warp w covers the 32 queries 32 (w / 4) .. of the block); warps 8-11 drain
// dQ^T (thread = one of the CTA's 128 head-dim columns) through a staging
// buffer, 16 query rows at a time, each chunk added to the CTA's half of the
// dQacc rows by one 2-D tensor bulk reduction; warp 12 issues the
// MMAs; warp 13 issues the TMA loads.  Every wait is bounded.
#pragma once

#include "bwd_kernel.cuh"

namespace fa {

struct Bwd256Cfg {
  static constexpr int D = 256;
  static constexpr int DH = 128;               // head-dim columns a CTA owns
  static constexpr int BN = 128;               // keys per CTA
  static constexpr int BM = 64;                // queries per iteration
  static constexpr int THREADS = 448;
  static constexpr int PDS_THREADS = 256;
  static constexpr int DRAIN_THREADS = 128;
  // Register split as in the head dim 128 kernel: 256 * 144 + 128 * 80 + 64 * 112
  // = 54272 <= 448 * 128; per sub-partition 2 * 144 + 80 + 112 = 480 <= 512.
  static constexpr int LAUNCH_REGS = 128;
  static constexpr int KREG = 128 * 128;       // one 64-column SW128 region of a 128-row tile (K, V, dS)
  static constexpr int QREG = 64 * 128;        // one 64-column SW128 region of a 64-row tile (Q, dO)
  static constexpr int KV_TILE = 4 * KREG;     // 128 x 256 bf16
  static constexpr int HALF = 2 * QREG;        // 64 x 128 bf16: one d-half of a Q or dO block
  static constexpr int OFF_K = 0, OFF_V = KV_TILE;
  static constexpr int OFF_Q_OWN = 2 * KV_TILE, OFF_Q_OTH = OFF_Q_OWN + HALF;
  static constexpr int OFF_DO_OWN = OFF_Q_OTH + HALF, OFF_DO_OTH = OFF_DO_OWN + HALF;
  static constexpr int OFF_DS = OFF_DO_OTH + HALF;            // dS, [key][query]: one 128-row region
  static constexpr int CHUNK_ROWS = 16;                       // query rows per dQ reduction (tm_dq's box)
  static constexpr int OFF_STG = OFF_DS + KREG;               // two dQ chunks, [row][owned d] fp32
  static constexpr int STG_BYTES = 2 * CHUNK_ROWS * DH * 4;
  static constexpr int OFF_VEC = OFF_STG + STG_BYTES;         // lse2[BM] then D[BM]
  static constexpr int VEC_BYTES = 2 * BM * 4;
  static constexpr int OFF_BAR = OFF_VEC + VEC_BYTES;
  static constexpr int N_BARS = 20;
  static constexpr int OFF_MISC = OFF_BAR + 8 * N_BARS;
  static constexpr int USED = OFF_MISC + 16;
  static constexpr int SMEM_BYTES = USED + 1024;              // + room to round the base up to 1 KB
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t T_DV = 0, T_DK = 128, T_S = 256, T_DP = 320, T_DQ = 384, T_P = 448;
  static constexpr uint32_t IDESC_SD = idesc_bf16_f32(128, BM, false, false);   // S^T, dP^T
  static constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, DH, false, true);    // dV (A in TMEM), dK
  static constexpr uint32_t IDESC_Q = idesc_bf16_f32(128, BM, true, true);      // dQ^T
};
static_assert(Bwd256Cfg::SMEM_BYTES <= 232448, "shared memory plan exceeds the per-block maximum");
static_assert(Bwd256Cfg::T_P + 32 <= Bwd256Cfg::TMEM_COLS, "tensor memory plan");
static_assert(Bwd256Cfg::PDS_THREADS * 144 + Bwd256Cfg::DRAIN_THREADS * 80 + 64 * 112 <=
                  Bwd256Cfg::THREADS * Bwd256Cfg::LAUNCH_REGS,
              "register split exceeds the registers the block launches with");
// setmaxnreg.inc takes registers freed in its own sub-partition: in sub-partitions
// 2 and 3 two P/dS warps (+16 each) against one drain warp (-48)
static_assert(2 * (144 - Bwd256Cfg::LAUNCH_REGS) <= Bwd256Cfg::LAUNCH_REGS - 80,
              "register split does not balance within a sub-partition");

// Work item x -> (key/value head bh, key block kb, owned half c).  The two halves
// of a key block are neighbours, so they read the same K, V, Q and dO from L2.
__host__ __device__ __forceinline__ void bwd256_decode(const BwdArgs& a, int x, int& bh, int& kb, int& c) {
  c = x & 1;
  bwd_decode(a, x >> 1, bh, kb);
}

template <bool PACKED>
__global__ void __launch_bounds__(Bwd256Cfg::THREADS, 1)
fa_bwd256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                 const __grid_constant__ CUtensorMap tm_dq, const BwdArgs args) {
  using C = Bwd256Cfg;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  int bh, kb, own;
  bwd256_decode(args, static_cast<int>(blockIdx.x), bh, kb, own);
  const int oth = own ^ 1;
  const int b = bh / args.L.H_kv, h_kv = bh - b * args.L.H_kv;
  const SeqSpan sp = seq_span<PACKED>(args.L, b, args.status);
  const int k0 = kb * C::BN;
  if (k0 >= sp.nk) return;
  const int off = sp.nk - sp.nq;                     // bottom-right causal alignment
  const int n_qb = (sp.nq + C::BM - 1) / C::BM;
  const int i_begin = args.causal ? max(0, k0 - off) / C::BM : 0;
  const int n_per = max(0, n_qb - i_begin);
  const int n_iter = n_per * args.group;
  const int col0 = own * C::DH;                      // first head-dim column this CTA owns
  if (n_iter == 0) {                                 // no query sees these keys: dK = dV = 0
    const int nk = min(C::BN, sp.nk - k0);
    for (int e = threadIdx.x; e < nk * (C::DH / 8); e += blockDim.x) {
      const int r = e / (C::DH / 8), cc = col0 + (e % (C::DH / 8)) * 8;
      *reinterpret_cast<uint4*>(args.dk + row_offset(args.sdk, sp.bc, h_kv, sp.k0 + k0 + r) + cc) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(args.dv + row_offset(args.sdv, sp.bc, h_kv, sp.k0 + k0 + r) + cc) = make_uint4(0, 0, 0, 0);
    }
    return;
  }
  auto q_head = [&](int it) { return h_kv * args.group + it / n_per; };
  auto q_row0 = [&](int it) { return (i_begin + it % n_per) * C::BM; };
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  if (pad + C::USED > static_cast<uint32_t>(C::SMEM_BYTES)) {
    if (threadIdx.x == 0) atomicOr(args.status, DEV_SMEM);
    return;
  }
  uint8_t* smem = smem_raw + pad;
  const uint32_t sbase = raw + pad;
  const uint32_t sK = sbase + C::OFF_K, sV = sbase + C::OFF_V, sDS = sbase + C::OFF_DS;
  const uint32_t sQown = sbase + C::OFF_Q_OWN, sQoth = sbase + C::OFF_Q_OTH;
  const uint32_t sDOown = sbase + C::OFF_DO_OWN, sDOoth = sbase + C::OFF_DO_OTH;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  const uint32_t b_kv_full = bar(0);
  const uint32_t b_qoth_full = bar(1), b_qoth_empty = bar(2);
  const uint32_t b_qown_full = bar(3), b_qown_empty = bar(4);    // with the lse2 / D vectors
  const uint32_t b_dooth_full = bar(5), b_dooth_empty = bar(6);
  const uint32_t b_doown_full = bar(7), b_doown_empty = bar(8);
  const uint32_t b_s_full = bar(9), b_s_free = bar(10);
  const uint32_t b_dp_full = bar(11), b_dp_free = bar(12);
  const uint32_t b_p_ready = bar(13), b_p_free = bar(14);
  const uint32_t b_ds_ready = bar(15), b_ds_free = bar(16);
  const uint32_t b_dq_full = bar(17), b_dq_free = bar(18);
  const uint32_t b_dkv_done = bar(19);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC + 4);
  uint64_t* drain_bar = reinterpret_cast<uint64_t*>(smem + C::OFF_MISC + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *abort_flag = 0u;
    for (int i = 0; i <= 9; ++i) mbar_init(bar(i), 1);   // loads (expect_tx) and s_full
    mbar_init(b_s_free, C::PDS_THREADS);
    mbar_init(b_dp_full, 1);
    mbar_init(b_dp_free, C::PDS_THREADS);
    mbar_init(b_p_ready, C::PDS_THREADS);
    mbar_init(b_p_free, 1);
    mbar_init(b_ds_ready, C::PDS_THREADS);
    mbar_init(b_ds_free, 1);
    mbar_init(b_dq_full, 1);
    mbar_init(b_dq_free, C::DRAIN_THREADS);
    mbar_init(b_dkv_done, 1);
    mbar_init(smem_u32(drain_bar), 1);
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
      // last iteration whose load was issued into each buffer (for the drain on failure)
      int last_qoth = -1, last_qown = -1, last_dooth = -1, last_doown = -1;
      mbar_expect_tx(b_kv_full, 2 * C::KV_TILE);
      for (int r = 0; r < 4; ++r) {
        tma_load_4d(sK + r * C::KREG, &tm_k, b_kv_full, r * 64, sp.k0 + k0, h_kv, sp.bc);
        tma_load_4d(sV + r * C::KREG, &tm_v, b_kv_full, r * 64, sp.k0 + k0, h_kv, sp.bc);
      }
      for (int it = 0; it < n_iter; ++it) {
        const uint32_t pp = (static_cast<uint32_t>(it) - 1u) & 1u;   // parity of the previous block's release
        const int q0 = q_row0(it);
        const int hq = q_head(it);
        // the halves not owned are released first (after S^T, dP^T), then dO's owned half (after dV)
        if (it > 0 && !mbar_wait(b_qoth_empty, pp, ctl)) { ok = false; break; }
        mbar_expect_tx(b_qoth_full, C::HALF);
        for (int r = 0; r < 2; ++r)
          tma_load_4d(sQoth + r * C::QREG, &tm_q, b_qoth_full, (2 * oth + r) * 64, sp.q0 + q0, hq, sp.bc);
        last_qoth = it;
        if (it > 0 && !mbar_wait(b_dooth_empty, pp, ctl)) { ok = false; break; }
        mbar_expect_tx(b_dooth_full, C::HALF);
        for (int r = 0; r < 2; ++r)
          tma_load_4d(sDOoth + r * C::QREG, &tm_do, b_dooth_full, (2 * oth + r) * 64, sp.q0 + q0, hq, sp.bc);
        last_dooth = it;
        if (it > 0 && !mbar_wait(b_doown_empty, pp, ctl)) { ok = false; break; }
        mbar_expect_tx(b_doown_full, C::HALF);
        for (int r = 0; r < 2; ++r)
          tma_load_4d(sDOown + r * C::QREG, &tm_do, b_doown_full, (2 * own + r) * 64, sp.q0 + q0, hq, sp.bc);
        last_doown = it;
        if (it > 0 && !mbar_wait(b_qown_empty, pp, ctl)) { ok = false; break; }
        mbar_expect_tx(b_qown_full, C::HALF + C::VEC_BYTES);
        for (int r = 0; r < 2; ++r)
          tma_load_4d(sQown + r * C::QREG, &tm_q, b_qown_full, (2 * own + r) * 64, sp.q0 + q0, hq, sp.bc);
        const size_t voff = (static_cast<size_t>(b) * args.L.H + hq) * args.Np + q0;
        bulk_load(sbase + C::OFF_VEC, args.lse2 + voff, C::BM * 4, b_qown_full);
        bulk_load(sbase + C::OFF_VEC + C::BM * 4, args.dvec + voff, C::BM * 4, b_qown_full);
        last_qown = it;
      }
      if (!ok) {       // let the loads in flight land before the CTA exits
        mbar_wait_quiet(b_kv_full, 0, 200000000ull);
        if (last_qoth >= 0) mbar_wait_quiet(b_qoth_full, last_qoth & 1, 200000000ull);
        if (last_dooth >= 0) mbar_wait_quiet(b_dooth_full, last_dooth & 1, 200000000ull);
        if (last_doown >= 0) mbar_wait_quiet(b_doown_full, last_doown & 1, 200000000ull);
        if (last_qown >= 0) mbar_wait_quiet(b_qown_full, last_qown & 1, 200000000ull);
      }
    }
  } else if (warp == 12) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop (its operands are warp-uniform) and one
    // elected lane issues each MMA and commit: measured faster than a loop run
    // by lane 0 alone.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 112;");
    {
      // K-major operands advance 32 B per K step inside a 128-byte row and switch
      // region every four steps; MN-major operands advance 16 rows (2 KB).
      const uint64_t dK_k = sdesc_sw128(sK, 16, 1024), dV_k = sdesc_sw128(sV, 16, 1024);
      const uint64_t dQoth_k = sdesc_sw128(sQoth, 16, 1024), dQown_k = sdesc_sw128(sQown, 16, 1024);
      const uint64_t dDOoth_k = sdesc_sw128(sDOoth, 16, 1024), dDOown_k = sdesc_sw128(sDOown, 16, 1024);
      const uint64_t dQown_mn = sdesc_sw128(sQown, C::QREG, 1024), dDOown_mn = sdesc_sw128(sDOown, C::QREG, 1024);
      const uint64_t dKown_mn = sdesc_sw128(sK + 2 * own * C::KREG, C::KREG, 1024);
      const uint64_t dDS_k = sdesc_sw128(sDS, 16, 1024), dDS_mn = sdesc_sw128(sDS, C::KREG, 1024);
      // K step kk (0..7) inside one d-half: of the 128-row K / V tiles, of the 64-row Q / dO halves
      auto kv_step = [](int half, int kk) {
        return static_cast<uint64_t>(((2 * half + (kk >> 2)) * C::KREG + (kk & 3) * 32) >> 4);
      };
      auto qh_step = [](int kk) { return static_cast<uint64_t>(((kk >> 2) * C::QREG + (kk & 3) * 32) >> 4); };
      auto mn_step = [](int kk) { return static_cast<uint64_t>((kk * 2048) >> 4); };
      // S^T or dP^T over the d-half `half` (A = K or V rows, B = that half of Q or dO)
      auto issue_sd = [&](uint32_t d_tmem, uint64_t a, uint64_t bq, int half, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ss_elect(d_tmem, a + kv_step(half, kk), bq + qh_step(kk), C::IDESC_SD, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait_warp(b_kv_full, 0, ctl);
      for (int it = 0; it < n_iter && ok; ++it) {
        const uint32_t ph = static_cast<uint32_t>(it) & 1u, pp = ph ^ 1u;
        // ---- S^T = K Q^T: the early (not owned) half of d first
        if (it > 0 && !mbar_wait_warp(b_s_free, pp, ctl)) { ok = false; break; }
        if (!mbar_wait_warp(b_qoth_full, ph, ctl)) { ok = false; break; }
        tc_fence_after();
        issue_sd(tmem + C::T_S, dK_k, dQoth_k, oth, false);
        umma_commit_elect(b_qoth_empty);
        if (!mbar_wait_warp(b_qown_full, ph, ctl)) { ok = false; break; }
        tc_fence_after();
        issue_sd(tmem + C::T_S, dK_k, dQown_k, own, true);
        umma_commit_elect(b_s_full);
        // ---- dP^T = V dO^T
        if (it > 0 && !mbar_wait_warp(b_dp_free, pp, ctl)) { ok = false; break; }
        if (!mbar_wait_warp(b_dooth_full, ph, ctl)) { ok = false; break; }
        tc_fence_after();
        issue_sd(tmem + C::T_DP, dV_k, dDOoth_k, oth, false);
        umma_commit_elect(b_dooth_empty);
        if (!mbar_wait_warp(b_doown_full, ph, ctl)) { ok = false; break; }
        tc_fence_after();
        issue_sd(tmem + C::T_DP, dV_k, dDOown_k, own, true);
        umma_commit_elect(b_dp_full);
        // ---- dV_c += P^T dO_c (A = P^T in TMEM, 8 packed columns per 16 queries)
        if (!mbar_wait_warp(b_p_ready, ph, ctl)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BM / 16; ++kk)
          umma_ts_elect(tmem + C::T_DV, tmem + C::T_P + 8 * kk, dDOown_mn + mn_step(kk), C::IDESC_KV,
                  (it > 0 || kk > 0) ? 1u : 0u);
        umma_commit_elect(b_doown_empty);
        umma_commit_elect(b_p_free);
        // ---- dK_c += dS^T Q_c, then dQ^T_c = K_c^T dS^T
        if (!mbar_wait_warp(b_ds_ready, ph, ctl)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BM / 16; ++kk)
          umma_ss_elect(tmem + C::T_DK, dDS_k + static_cast<uint64_t>((kk * 32) >> 4), dQown_mn + mn_step(kk), C::IDESC_KV,
                  (it > 0 || kk > 0) ? 1u : 0u);
        umma_commit_elect(b_qown_empty);
        if (it > 0 && !mbar_wait_warp(b_dq_free, pp, ctl)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          umma_ss_elect(tmem + C::T_DQ, dKown_mn + mn_step(kk), dDS_mn + mn_step(kk), C::IDESC_Q, kk > 0 ? 1u : 0u);
        umma_commit_elect(b_dq_full);
        umma_commit_elect(b_ds_free);
      }
      if (ok) umma_commit_elect(b_dkv_done);
      umma_commit_elect(smem_u32(drain_bar));
      mbar_wait_quiet(smem_u32(drain_bar), 0, 200000000ull);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ P / dS warps (thread = key, 32 queries)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 144;");
    const int quarter = warp & 3;
    const int ch = warp >> 2;                       // queries 32 ch .. 32 ch + 31 of the block
    const int rloc = quarter * 32 + lane;           // key row in the block == TMEM lane
    const int key = k0 + rloc;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::T_S + 32 * ch;
    const uint32_t tDP = tmem + lane_off + C::T_DP + 32 * ch;
    const uint32_t tP = tmem + lane_off + C::T_P + 16 * ch;
    const float c2 = args.scale_log2;
    const bool key_ok = key < sp.nk;
    // this thread's 64 bytes of its dS row: 16-byte chunks 4 ch .. 4 ch + 3 of row
    // rloc, chunk j stored at chunk j ^ (row & 7) (128-byte swizzle)
    uint8_t* prow = smem + C::OFF_DS + rloc * 128;
    const int sw = rloc & 7;
    const float* lse2 = reinterpret_cast<const float*>(smem + C::OFF_VEC) + 32 * ch;
    const float* dvec = lse2 + C::BM;
    bool ok = true;
    for (int it = 0; it < n_iter; ++it) {
      const uint32_t ph = static_cast<uint32_t>(it) & 1u, pp = ph ^ 1u;
      const int q0 = q_row0(it);
      if (!mbar_wait_warp(b_qown_full, ph, ctl)) { ok = false; break; }   // lse2, D of this block
      if (!mbar_wait_warp(b_s_full, ph, ctl)) { ok = false; break; }
      tc_fence_after();
      float p[32];
      {
        uint32_t ra[32];
        tmem_ld32(tS, ra);
        tmem_wait_ld();
        reg_fence32(ra);
        tc_fence_before();
        mbar_arrive(b_s_free);
        // 2^x on the special-function unit: at d = 256 each exponential comes with
        // twice the tensor work of d = 128, so that unit is not the limit here
        const float2 c2v = make_float2(c2, c2);
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c);
          const float2 xa = ffma2(make_float2(__uint_as_float(ra[c]), __uint_as_float(ra[c + 1])), c2v,
                                  make_float2(-l4.x, -l4.y));
          const float2 xb = ffma2(make_float2(__uint_as_float(ra[c + 2]), __uint_as_float(ra[c + 3])), c2v,
                                  make_float2(-l4.z, -l4.w));
          p[c] = ex2_approx(xa.x);
          p[c + 1] = ex2_approx(xa.y);
          p[c + 2] = ex2_approx(xb.x);
          p[c + 3] = ex2_approx(xb.y);
        }
      }
      // keys past the sequence end, and (causal) queries that do not see this key: P = 0
      const int cut = !key_ok ? C::BM : (args.causal ? key - off - q0 : 0);   // block columns c < cut are masked
      if (cut > 32 * ch) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (32 * ch + c < cut) p[c] = 0.f;
      }
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(p[2 * c], p[2 * c + 1]);
      if (it > 0 && !mbar_wait_warp(b_p_free, pp, ctl)) { ok = false; break; }   // dV_{i-1} read P_{i-1}
      tc_fence_after();
      tmem_st16(tP, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(b_p_ready);
      // dS = P (dP - D)
      if (!mbar_wait_warp(b_dp_full, ph, ctl)) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t ra[32];
        tmem_ld32(tDP, ra);
        tmem_wait_ld();
        reg_fence32(ra);
        tc_fence_before();
        mbar_arrive(b_dp_free);
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 d4 = *reinterpret_cast<const float4*>(dvec + c);
          const float2 ga = fmul2(make_float2(p[c], p[c + 1]),
                                  fsub2(make_float2(__uint_as_float(ra[c]), __uint_as_float(ra[c + 1])),
                                        make_float2(d4.x, d4.y)));
          const float2 gb = fmul2(make_float2(p[c + 2], p[c + 3]),
                                  fsub2(make_float2(__uint_as_float(ra[c + 2]), __uint_as_float(ra[c + 3])),
                                        make_float2(d4.z, d4.w)));
          pk[c >> 1] = pack_bf16x2(ga.x, ga.y);
          pk[(c >> 1) + 1] = pack_bf16x2(gb.x, gb.y);
        }
      }
      if (it > 0 && !mbar_wait_warp(b_ds_free, pp, ctl)) { ok = false; break; }   // dK_{i-1}, dQ_{i-1} read dS
#pragma unroll
      for (int j = 0; j < 4; ++j)
        *reinterpret_cast<uint4*>(prow + (((4 * ch + j) ^ sw) << 4)) =
            make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
      fence_proxy_async_smem();
      mbar_arrive(b_ds_ready);
    }
    // ---- epilogue: this thread's 64 columns of its dV and dK rows (of the CTA's half) -> global
    if (ok && mbar_wait_warp(b_dkv_done, 0, ctl)) {
      tc_fence_after();
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t tsrc = tmem + lane_off + (which ? C::T_DK : C::T_DV) + 64 * ch;
        __nv_bfloat16* dst = which ? args.dk + row_offset(args.sdk, sp.bc, h_kv, sp.k0 + key) + col0 + 64 * ch
                                   : args.dv + row_offset(args.sdv, sp.bc, h_kv, sp.k0 + key) + col0 + 64 * ch;
        const float mul = which ? args.scale : 1.0f;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t v[32];
          tmem_ld32(tsrc + cc * 32, v);
          tmem_wait_ld();
          reg_fence32(v);
          if (key_ok) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + cc * 32);
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
    // ------------------------------------------------------------ dQ drain (thread = owned head-dim column)
    // Chunks of 16 query rows go row-major ([row][owned d], fp32) into one of two
    // staging buffers and one thread adds each to dQacc with a tensor bulk
    // reduction of the map's 128 x 16 box.  Rows past the sequence end are
    // included (their dS, so their dQ, is exactly zero: P = 2^-inf there) and
    // rows past the accumulator are not written.  The wait for each block ends
    // in a vote of the four drain warps, so none is left at a named barrier.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 80;");
    const int dl = (warp - 8) * 32 + lane;
    const bool issuer = dl == 0;
    const uint32_t tDQ = tmem + (static_cast<uint32_t>((warp - 8) * 32) << 16) + C::T_DQ;
    float* stg = reinterpret_cast<float*>(smem + C::OFF_STG);
    int last_buf = 1;                                  // staging buffer of the newest reduction
    for (int it = 0; it < n_iter; ++it) {
      if (!named_bar_and(1, C::DRAIN_THREADS, mbar_wait_warp(b_dq_full, static_cast<uint32_t>(it) & 1u, ctl))) break;
      tc_fence_after();
      const int q0 = q_row0(it);
      const int nq = min(C::BM, sp.nq - q0);
      uint32_t r[64];
      tmem_ld32(tDQ, *reinterpret_cast<uint32_t(*)[32]>(r));
      tmem_ld32(tDQ + 32, *reinterpret_cast<uint32_t(*)[32]>(r + 32));
      tmem_wait_ld();
      reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(r));
      reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(r + 32));
      tc_fence_before();
      mbar_arrive(b_dq_free);
#pragma unroll
      for (int c = 0; c < C::BM / C::CHUNK_ROWS; ++c) {   // chunk c: queries 16c .. 16c + 15 of the block
        if (C::CHUNK_ROWS * c >= nq) break;               // uniform over the drain warps
        // the reduction that used this buffer before has read it: the newest one
        // when a ragged block ended on this buffer, else the one before it
        if (issuer) {
          if ((c & 1) == last_buf) bulk_wait_read<0>();
          else bulk_wait_read<1>();
        }
        last_buf = c & 1;
        named_bar_sync(1, C::DRAIN_THREADS);
        float* buf = stg + (c & 1) * C::CHUNK_ROWS * C::DH;
#pragma unroll
        for (int j = 0; j < C::CHUNK_ROWS; ++j) buf[j * C::DH + dl] = __uint_as_float(r[C::CHUNK_ROWS * c + j]);
        fence_proxy_async_smem();
        named_bar_sync(1, C::DRAIN_THREADS);
        if (issuer) {
          const long long row = row_index<PACKED>(args.L, sp, q_head(it), q0 + C::CHUNK_ROWS * c);
          tma_reduce_add_2d(&tm_dq, sbase + C::OFF_STG + (c & 1) * C::CHUNK_ROWS * C::DH * 4, col0,
                            static_cast<int>(row));
          bulk_commit();
        }
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
