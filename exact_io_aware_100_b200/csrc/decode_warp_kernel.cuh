// Decode attention with warp-independent key tiles, for at most four query rows
// per key/value head (e.g. one new token for a set of four query heads).
//
// Same result as decode_kernel.cuh (the last N_q query positions against an N_k
// key cache, keys split across CTAs, the split partials combined by the softmax
// merge of the unite.ai page "Flash Attention: Rivoluzionando l'Efficienza dei
// Modelli Transformer", "La Matematica dietro Flash Attention"; the decode
// workload of the gist.science FlashAttention-V page), organised so that no
// block barrier sits in the key loop:
//
//  * each warp of a CTA streams its own 16-key K / V tiles (tiles w, w + 4, ...
//    of the CTA's split) through a private three-stage TMA ring and keeps its
//    own online softmax (row max m, row sum l) for the four rows;
//  * lane = (key slot sk = lane / 8, head-dim group dg = lane % 8): the lane
//    keeps the four query rows' 16 columns 16 dg .. 16 dg + 15 in registers and
//    the four rows' partial output over the same columns; per pass it takes
//    key 4 p + sk of the tile, forms four partial dot products over its 16
//    columns and reduces them over the eight dg lanes with a butterfly that
//    leaves row dg / 2's score in the lane (four shuffles for four rows);
//  * the tile's probabilities go through a 256-byte per-warp buffer so every
//    lane reads the four rows' p of its keys with one 16-byte load per key;
//    O is rescaled only when a row's max grows by more than 2^8 (exp2 units);
//  * at the end of the split the warps' (m, l, O) are merged in shared memory
//    (the softmax merge) into the split's normalised partial and its lse, the
//    format fa_decode_merge_kernel combines.
// HBM-bound work on the CUDA cores (packed fp32 FMAs); every wait is bounded.
#pragma once

#include "decode_kernel.cuh"

namespace fa {

struct DecWCfg {
  static constexpr int D = 128;
  static constexpr int KT = 16;                  // keys per tile
  static constexpr int R = 4;                    // query rows per CTA
  static constexpr int WARPS = 4;
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int STAGES = 3;
  static constexpr int KREG = KT * 128;          // one 64-column swizzle region of a 16-row tile (2 KB)
  static constexpr int TILE = 2 * KREG;          // 16 x 128 bf16 (4 KB)
  static constexpr int STAGE = 2 * TILE;         // K then V
  static constexpr int WARP_RING = STAGES * STAGE;
  static constexpr int OFF_RING = 0;             // per warp: STAGES stages (1 KB aligned)
  static constexpr int OFF_P = WARPS * WARP_RING;                  // per warp: p [KT][R] fp32 + alpha [R]
  static constexpr int P_BYTES = (KT * R + R) * 4;
  static constexpr int OFF_BAR = OFF_P + WARPS * P_BYTES;          // per warp: STAGES full barriers
  static constexpr int OFF_MISC = OFF_BAR + 8 * WARPS * STAGES;    // abort flag
  static constexpr int USED = OFF_MISC + 16;
  static constexpr int SMEM_BYTES = USED + 1024;
  // the end-of-split merge reuses the rings: per warp O [R][D] fp32, then m [R], l [R]
  static constexpr int MERGE_BYTES = WARPS * (R * D + 2 * R) * 4;
};
static_assert(DecWCfg::MERGE_BYTES <= DecWCfg::OFF_P, "merge buffer fits in the rings");
static_assert(2 * DecWCfg::SMEM_BYTES <= 232448, "two CTAs per SM");

__global__ void __launch_bounds__(DecWCfg::THREADS, 2)
fa_decode_warp_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const DecArgs a) {
  using C = DecWCfg;
  constexpr int D = C::D, R = C::R;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sk = lane >> 3, dg = lane & 7;
  const int split = blockIdx.x;
  const int bhkv = blockIdx.y;
  const int h_kv_count = a.heads / a.group;
  const int bhq0 = (bhkv / h_kv_count) * a.heads + (bhkv % h_kv_count) * a.group;   // first query head of the set
  const int rows = a.group * a.Lq;                 // <= R
  const int k_begin = split * a.split_keys;
  const int k_end = min(k_begin + a.split_keys, a.Nk);
  const int n_tiles = (k_end - k_begin + C::KT - 1) / C::KT;
  const int my_tiles = n_tiles > warp ? (n_tiles - warp + C::WARPS - 1) / C::WARPS : 0;   // tiles warp, warp + 4, ...
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC);
  const uint32_t bar0 = sbase + C::OFF_BAR + 8 * C::STAGES * warp;
  const uint32_t ring = sbase + C::OFF_RING + warp * C::WARP_RING;
  float* pbuf = reinterpret_cast<float*>(smem + C::OFF_P + warp * C::P_BYTES);   // [KT][R] then alpha [R]

  if (lane == 0) {
    for (int st = 0; st < C::STAGES; ++st) mbar_init(bar0 + 8 * st, 1);
    fence_mbar_init();
  }
  if (tid == 0) *abort_flag = 0u;
  __syncthreads();
  const WaitCtl ctl{abort_flag, a.status, a.wait_limit_ns};
  auto issue = [&](int i) {          // this warp's i-th tile into stage i % STAGES (lane 0)
    const uint32_t st = ring + (i % C::STAGES) * C::STAGE;
    const uint32_t bar = bar0 + 8 * (i % C::STAGES);
    mbar_expect_tx(bar, C::STAGE);
    const int y = k_begin + (warp + C::WARPS * i) * C::KT;
    for (int r = 0; r < 2; ++r) {
      tma_load_3d(st + r * C::KREG, &tm_k, bar, r * 64, y, bhkv);
      tma_load_3d(st + C::TILE + r * C::KREG, &tm_v, bar, r * 64, y, bhkv);
    }
  };
  if (lane == 0)
    for (int i = 0; i < C::STAGES && i < my_tiles; ++i) issue(i);

  // the four query rows' columns 16 dg .. 16 dg + 15 (rows >= rows() are zero)
  float2 qf[R][8];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (r < rows) {
      const int hq = bhq0 + r / a.Lq, i = r % a.Lq;
      const uint4* src = reinterpret_cast<const uint4*>(a.q + (static_cast<size_t>(hq) * a.Lq + i) * D + 16 * dg);
      const uint4 w0 = __ldg(src), w1 = __ldg(src + 1);
      qf[r][0] = bf16x2_to_float2(w0.x); qf[r][1] = bf16x2_to_float2(w0.y);
      qf[r][2] = bf16x2_to_float2(w0.z); qf[r][3] = bf16x2_to_float2(w0.w);
      qf[r][4] = bf16x2_to_float2(w1.x); qf[r][5] = bf16x2_to_float2(w1.y);
      qf[r][6] = bf16x2_to_float2(w1.z); qf[r][7] = bf16x2_to_float2(w1.w);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[r][e] = make_float2(0.f, 0.f);
    }
  }
  const float c2 = a.scale_log2;
  const int my_row = dg >> 1;                    // the row whose score the butterfly leaves in this lane
  // causal limit of my_row: key positions <= lim are visible
  const int lim = a.causal ? a.Nk - a.Lq + my_row % a.Lq : a.Nk - 1;
  float m = -INFINITY, l = 0.f;                  // my_row's running max and sum
  float2 acc[R][8];                              // partial O, rows x columns 16 dg ..
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[r][e] = make_float2(0.f, 0.f);
  // this lane's two 16-byte chunks of a 128-byte K / V row: region dg / 4, chunks 2 (dg % 4), + 1
  const uint32_t col_reg = (dg >> 2) * C::KREG;
  const int ch0 = (dg & 3) * 2;

  bool ok = true;
  int i_fail = my_tiles;
  for (int i = 0; i < my_tiles; ++i) {
    if (!mbar_wait_warp(bar0 + 8 * (i % C::STAGES), (i / C::STAGES) & 1, ctl)) { ok = false; i_fail = i; break; }
    const uint8_t* st = smem + C::OFF_RING + warp * C::WARP_RING + (i % C::STAGES) * C::STAGE;
    const int kt0 = k_begin + (warp + C::WARPS * i) * C::KT;
    // ---- scores: four passes, key 4 p + sk; my_row's score of each key stays in sc[p]
    float sc[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int key = 4 * p + sk;
      const uint8_t* krow = st + col_reg + key * 128;
      const uint4 w0 = *reinterpret_cast<const uint4*>(krow + (((ch0) ^ (key & 7)) << 4));
      const uint4 w1 = *reinterpret_cast<const uint4*>(krow + (((ch0 + 1) ^ (key & 7)) << 4));
      const float2 kf[8] = {bf16x2_to_float2(w0.x), bf16x2_to_float2(w0.y), bf16x2_to_float2(w0.z),
                            bf16x2_to_float2(w0.w), bf16x2_to_float2(w1.x), bf16x2_to_float2(w1.y),
                            bf16x2_to_float2(w1.z), bf16x2_to_float2(w1.w)};
      float part[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 8; ++e) s2 = ffma2(qf[r][e], kf[e], s2);
        part[r] = s2.x + s2.y;
      }
      // butterfly over the eight dg lanes: after it, lane dg holds row dg / 2 summed over all 128 columns
      const bool b2 = (dg & 4) != 0, b1 = (dg & 2) != 0;
      const float x0 = __shfl_xor_sync(0xffffffffu, b2 ? part[0] : part[2], 4);
      const float x1 = __shfl_xor_sync(0xffffffffu, b2 ? part[1] : part[3], 4);
      const float k0 = (b2 ? part[2] : part[0]) + x0;          // rows 2 b2, 2 b2 + 1
      const float k1 = (b2 ? part[3] : part[1]) + x1;
      float v = (b1 ? k1 : k0) + __shfl_xor_sync(0xffffffffu, b1 ? k0 : k1, 2);   // row 2 b2 + b1
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      const int pos = kt0 + key;
      sc[p] = (my_row < rows && pos < k_end && pos <= lim) ? v : -INFINITY;
    }
    // ---- online softmax of my_row over the tile's 16 keys (the 4 sk lanes x 4 passes)
    float tmax = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 8));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
    const float m_new = fmaxf(m, tmax);
    const bool need = (m_new - m) * c2 > 8.0f;   // false while the row has seen no key
    float alpha = 1.0f;
    if (need) {
      alpha = m_new == -INFINITY ? 1.0f : ex2_approx((m - m_new) * c2);   // 0 on the first visible key
      l *= alpha;
      m = m_new;
    }
    const float nb = m == -INFINITY ? 0.0f : m * c2;
    float pv[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) pv[p] = ex2_approx(fmaf(sc[p], c2, -nb));
    float ps = (pv[0] + pv[1]) + (pv[2] + pv[3]);
    ps += __shfl_xor_sync(0xffffffffu, ps, 8);
    ps += __shfl_xor_sync(0xffffffffu, ps, 16);
    l += ps;
    // p of (key, row) and each row's alpha to the warp's buffer (one writer per row: dg even)
    const bool any_rescale = __any_sync(0xffffffffu, need);
    if ((dg & 1) == 0) {
#pragma unroll
      for (int p = 0; p < 4; ++p) pbuf[(4 * p + sk) * R + my_row] = pv[p];
      if (sk == 0) pbuf[C::KT * R + my_row] = alpha;
    }
    __syncwarp();
    if (any_rescale) {
      const float4 al = *reinterpret_cast<const float4*>(pbuf + C::KT * R);
      const float alr[R] = {al.x, al.y, al.z, al.w};
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[r][e] = fmul2(acc[r][e], make_float2(alr[r], alr[r]));
    }
    // ---- P.V: keys 4 p + sk, columns 16 dg ..
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int key = 4 * p + sk;
      const uint8_t* vrow = st + C::TILE + col_reg + key * 128;
      const uint4 w0 = *reinterpret_cast<const uint4*>(vrow + (((ch0) ^ (key & 7)) << 4));
      const uint4 w1 = *reinterpret_cast<const uint4*>(vrow + (((ch0 + 1) ^ (key & 7)) << 4));
      const float2 vf[8] = {bf16x2_to_float2(w0.x), bf16x2_to_float2(w0.y), bf16x2_to_float2(w0.z),
                            bf16x2_to_float2(w0.w), bf16x2_to_float2(w1.x), bf16x2_to_float2(w1.y),
                            bf16x2_to_float2(w1.z), bf16x2_to_float2(w1.w)};
      const float4 p4 = *reinterpret_cast<const float4*>(pbuf + key * R);
      const float pr[R] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[r][e] = ffma2(make_float2(pr[r], pr[r]), vf[e], acc[r][e]);
    }
    __syncwarp();                                // every lane is done with the stage and the p buffer
    if (lane == 0 && i + C::STAGES < my_tiles) issue(i + C::STAGES);
  }
  if (!ok) {
    // let this warp's loads in flight land before the CTA exits (bounded)
    if (lane == 0)
      for (int i = i_fail; i < my_tiles && i < i_fail + C::STAGES; ++i)
        mbar_wait_quiet(bar0 + 8 * (i % C::STAGES), (i / C::STAGES) & 1, 200000000ull);
  }
  // ---- the warp's partial O: sum over the four key slots (same dg, every sk)
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      acc[r][e].x += __shfl_xor_sync(0xffffffffu, acc[r][e].x, 8);
      acc[r][e].y += __shfl_xor_sync(0xffffffffu, acc[r][e].y, 8);
      acc[r][e].x += __shfl_xor_sync(0xffffffffu, acc[r][e].x, 16);
      acc[r][e].y += __shfl_xor_sync(0xffffffffu, acc[r][e].y, 16);
    }
  __syncthreads();                                 // every warp is done with the rings
  if (!__syncthreads_or(!ok)) {
    // ---- merge the warps (softmax merge) in the ring area: per warp O [R][D], m [R], l [R]
    float* mo = reinterpret_cast<float*>(smem + C::OFF_RING);
    float* wo = mo + warp * (R * D + 2 * R);
    if (sk == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) *reinterpret_cast<float2*>(wo + r * D + 16 * dg + 2 * e) = acc[r][e];
    }
    if (sk == 0 && (dg & 1) == 0) {
      wo[R * D + my_row] = m;
      wo[R * D + R + my_row] = l;
    }
    __syncthreads();
    // thread = (row, 4 columns): 4 rows x 32 column groups = 128 threads
    const int r = tid >> 5, c4 = tid & 31;
    if (r < rows) {
      float mx = -INFINITY;
      for (int w = 0; w < C::WARPS; ++w) mx = fmaxf(mx, mo[w * (R * D + 2 * R) + R * D + r]);
      float lsum = 0.f;
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      if (mx != -INFINITY) {
        for (int w = 0; w < C::WARPS; ++w) {
          const float* ww = mo + w * (R * D + 2 * R);
          const float mw = ww[R * D + r];
          if (mw == -INFINITY) continue;
          const float f = ex2_approx((mw - mx) * c2);
          lsum = fmaf(f, ww[R * D + R + r], lsum);
          const float4 x = *reinterpret_cast<const float4*>(ww + r * D + 4 * c4);
          o.x = fmaf(f, x.x, o.x);
          o.y = fmaf(f, x.y, o.y);
          o.z = fmaf(f, x.z, o.z);
          o.w = fmaf(f, x.w, o.w);
        }
      }
      const int hq = bhq0 + r / a.Lq, qi = r % a.Lq;
      const size_t row = (static_cast<size_t>(split) * a.bh + hq) * a.Lq + qi;
      const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;
      *reinterpret_cast<float4*>(a.part_o + row * D + 4 * c4) = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
      if (c4 == 0) a.part_lse[row] = lsum > 0.f ? (mx * c2 + __log2f(lsum)) * 0.69314718055994531f : -INFINITY;
    }
  }
}

}  // namespace fa
