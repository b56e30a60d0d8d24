// Decode attention for sm_100a: a few queries (the last N_q positions) against
// a long key/value cache, with the keys split across CTAs and the partial
// results combined by the softmax merge.
//
// The merge is the one the unite.ai page "Flash Attention: Rivoluzionando
// l'Efficienza dei Modelli Transformer" gives in "La Matematica dietro Flash
// Attention": partial results over disjoint key sets combine through their
// maxima and sums; here each partial is kept normalised with its natural-log
// logsumexp, so  lse = ln sum_s e^{lse_s}  and  O = sum_s e^{lse_s - lse} O_s.
// The decode workload is the one the gist.science FlashAttention-V page times;
// grouped-query sets follow the nearauto.com FlashAttention-2 digest (one
// key/value head per set of query heads).
//
// Decoding reads every key and value once for a handful of query rows, so it is
// bound by HBM bandwidth, not by arithmetic: the kernel streams K / V tiles with
// TMA into shared memory and does the small products on the CUDA cores
// (fp32 FMAs) rather than shaping them into tensor-core tiles.
//
//  * fa_decode_kernel:  one CTA per (batch * key/value head, key split).  The
//    rows are the N_q queries of every query head of the key/value head's set
//    (at most 16 rows).  64-key tiles of K and V stream through a two-stage
//    TMA ring (128-byte swizzle, so per-lane shared reads are conflict free).
//    Warp w owns rows w and w + 8; for scores each lane takes two keys, for
//    P.V each lane four of the 128 output columns.  Writes the split's
//    normalised partial O (fp32) and its lse (-inf when no key is visible);
//  * fa_decode_merge_kernel:  one warp per query row, merges the splits.
#pragma once

#include "ptx.cuh"

namespace fa {

struct DecArgs {
  const __nv_bfloat16* q;   // [BH, Lq, 128]
  float* part_o;            // [splits, BH, Lq, 128] fp32, normalised per split
  float* part_lse;          // [splits, BH, Lq] natural log, -inf when the split saw no key
  __nv_bfloat16* o;         // [BH, Lq, 128]
  float* lse;               // [BH, Lq]
  uint32_t* status;
  int Lq, Nk;
  int heads, group;         // query heads per batch entry, query heads per key/value head
  int bh, bh_kv;            // B * H, B * H_kv
  int split_keys;           // keys per split (a multiple of 64)
  int n_splits;
  int causal;
  float scale_log2;
  unsigned long long wait_limit_ns;
};

struct DecCfg {
  static constexpr int D = 128;
  static constexpr int KT = 64;                  // keys per tile
  static constexpr int R_MAX = 16;               // query rows per CTA
  static constexpr int THREADS = 256;
  static constexpr int KREG = KT * 128;          // one 64-column swizzle region of a 64-row tile
  static constexpr int TILE = 2 * KREG;          // a 64 x 128 bf16 tile (16 KB)
  static constexpr int OFF_Q = 0;                // fp32 [R_MAX][D]
  static constexpr int OFF_ST = R_MAX * D * 4;   // two stages of K then V
  static constexpr int STAGE = 2 * TILE;
  static constexpr int OFF_BAR = OFF_ST + 2 * STAGE;
  static constexpr int OFF_MISC = OFF_BAR + 16;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;   // + alignment slack
};

// Splits for a cache of Nk keys and bh_kv key/value heads: about a thousand CTAs
// in total (several waves on any B200), each split a whole number of 64-key tiles.
__host__ __device__ inline int decode_splits(int bh_kv, int Nk, int* split_keys) {
  const int tiles = (Nk + DecCfg::KT - 1) / DecCfg::KT;
  int want = (1024 + bh_kv - 1) / bh_kv;
  if (want < 1) want = 1;
  if (want > tiles) want = tiles;
  const int tiles_per = (tiles + want - 1) / want;
  *split_keys = tiles_per * DecCfg::KT;
  return (tiles + tiles_per - 1) / tiles_per;
}

__global__ void __launch_bounds__(DecCfg::THREADS)
fa_decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                 const DecArgs a) {
  using C = DecCfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* sq = reinterpret_cast<float*>(smem + C::OFF_Q);
  const uint32_t b_full0 = sbase + C::OFF_BAR;
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x;
  const int bhkv = blockIdx.y;
  const int h_kv_count = a.heads / a.group;
  const int bhq0 = (bhkv / h_kv_count) * a.heads + (bhkv % h_kv_count) * a.group;   // first query head of the set
  const int R = a.group * a.Lq;
  const int k_begin = split * a.split_keys;
  const int k_end = min(k_begin + a.split_keys, a.Nk);
  const int n_tiles = (k_end - k_begin + C::KT - 1) / C::KT;

  if (tid == 0) {
    *abort_flag = 0u;
    mbar_init(b_full0, 1);
    mbar_init(b_full0 + 8, 1);
    fence_mbar_init();
  }
  // query rows (fp32), row r = (query head g of the set, position i); rows >= R are zero
  for (int idx = tid; idx < C::R_MAX * D; idx += C::THREADS) {
    const int r = idx / D, c = idx % D;
    float x = 0.f;
    if (r < R) {
      const int hq = bhq0 + r / a.Lq, i = r % a.Lq;
      x = __bfloat162float(a.q[(static_cast<size_t>(hq) * a.Lq + i) * D + c]);
    }
    sq[idx] = x;
  }
  __syncthreads();
  const WaitCtl ctl{abort_flag, a.status, a.wait_limit_ns};
  auto issue = [&](int t) {         // tile t of this split into stage t % 2 (thread 0)
    const uint32_t st = sbase + C::OFF_ST + (t & 1) * C::STAGE;
    const uint32_t bar = b_full0 + 8 * (t & 1);
    mbar_expect_tx(bar, 2 * C::TILE);
    const int y = k_begin + t * C::KT;
    for (int r = 0; r < 2; ++r) {
      tma_load_3d(st + r * C::KREG, &tm_k, bar, r * 64, y, bhkv);
      tma_load_3d(st + C::TILE + r * C::KREG, &tm_v, bar, r * 64, y, bhkv);
    }
  };
  if (tid == 0) {
    if (n_tiles > 0) issue(0);
    if (n_tiles > 1) issue(1);
  }

  // this warp's rows and their causal limits (key positions <= lim are visible)
  const int ra = warp, rb = warp + 8;
  const bool va = ra < R, vb = rb < R;
  const int lim_a = a.causal ? a.Nk - a.Lq + ra % a.Lq : a.Nk - 1;
  const int lim_b = a.causal ? a.Nk - a.Lq + rb % a.Lq : a.Nk - 1;
  const float c2 = a.scale_log2;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
  float oa[4] = {0.f, 0.f, 0.f, 0.f}, ob[4] = {0.f, 0.f, 0.f, 0.f};
  bool ok = true;
  int t_fail = n_tiles;
  for (int t = 0; t < n_tiles; ++t) {
    ok = ok && mbar_wait(b_full0 + 8 * (t & 1), (t >> 1) & 1, ctl);
    if (!__syncthreads_and(ok)) { ok = false; t_fail = t; break; }   // every thread agrees before using the stage
    const uint8_t* st = smem + C::OFF_ST + (t & 1) * C::STAGE;
    const int kt0 = k_begin + t * C::KT;
    if (va) {
      // scores of rows ra, rb against keys lane and lane + 32
      float sa0 = 0.f, sa1 = 0.f, sb0 = 0.f, sb1 = 0.f;
      const int k0 = lane, k1 = lane + 32;
#pragma unroll
      for (int j = 0; j < 16; ++j) {        // 16-byte chunks along d
        const int region = j >> 3, c = j & 7;
        const uint4 w0 = *reinterpret_cast<const uint4*>(st + region * C::KREG + k0 * 128 + ((c ^ (k0 & 7)) << 4));
        const uint4 w1 = *reinterpret_cast<const uint4*>(st + region * C::KREG + k1 * 128 + ((c ^ (k1 & 7)) << 4));
        const uint32_t ka[4] = {w0.x, w0.y, w0.z, w0.w}, kb[4] = {w1.x, w1.y, w1.z, w1.w};
        const float4 qa0 = *reinterpret_cast<const float4*>(sq + ra * D + 8 * j);
        const float4 qa1 = *reinterpret_cast<const float4*>(sq + ra * D + 8 * j + 4);
        const float4 qb0 = *reinterpret_cast<const float4*>(sq + (vb ? rb : ra) * D + 8 * j);
        const float4 qb1 = *reinterpret_cast<const float4*>(sq + (vb ? rb : ra) * D + 8 * j + 4);
        const float qa[8] = {qa0.x, qa0.y, qa0.z, qa0.w, qa1.x, qa1.y, qa1.z, qa1.w};
        const float qb[8] = {qb0.x, qb0.y, qb0.z, qb0.w, qb1.x, qb1.y, qb1.z, qb1.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ka[e]));
          const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kb[e]));
          sa0 = fmaf(qa[2 * e], f0.x, fmaf(qa[2 * e + 1], f0.y, sa0));
          sa1 = fmaf(qa[2 * e], f1.x, fmaf(qa[2 * e + 1], f1.y, sa1));
          if (vb) {                          // warp-uniform: a second row only when the set has one
            sb0 = fmaf(qb[2 * e], f0.x, fmaf(qb[2 * e + 1], f0.y, sb0));
            sb1 = fmaf(qb[2 * e], f1.x, fmaf(qb[2 * e + 1], f1.y, sb1));
          }
        }
      }
      // mask: keys past the split (or the cache) and, causal, after the query's position
      const int p0 = kt0 + k0, p1 = kt0 + k1;
      if (p0 >= k_end || p0 > lim_a) sa0 = -INFINITY;
      if (p1 >= k_end || p1 > lim_a) sa1 = -INFINITY;
      if (!vb || p0 >= k_end || p0 > lim_b) sb0 = -INFINITY;
      if (!vb || p1 >= k_end || p1 > lim_b) sb1 = -INFINITY;
      // online softmax, per row, over the warp's 64 keys
      float ta = fmaxf(sa0, sa1), tb = fmaxf(sb0, sb1);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        ta = fmaxf(ta, __shfl_xor_sync(0xffffffffu, ta, off));
        tb = fmaxf(tb, __shfl_xor_sync(0xffffffffu, tb, off));
      }
      const float mna = fmaxf(m_a, ta), mnb = fmaxf(m_b, tb);
      // rows that have seen no visible key keep m = -inf and contribute nothing
      const float alpha_a = (mna == -INFINITY) ? 1.f : ex2_approx((m_a - mna) * c2);
      const float alpha_b = (mnb == -INFINITY) ? 1.f : ex2_approx((m_b - mnb) * c2);
      const float na = (mna == -INFINITY) ? 0.f : mna * c2, nb = (mnb == -INFINITY) ? 0.f : mnb * c2;
      const float pa0 = ex2_approx(fmaf(sa0, c2, -na)), pa1 = ex2_approx(fmaf(sa1, c2, -na));
      const float pb0 = ex2_approx(fmaf(sb0, c2, -nb)), pb1 = ex2_approx(fmaf(sb1, c2, -nb));
      float suma = pa0 + pa1, sumb = pb0 + pb1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        suma += __shfl_xor_sync(0xffffffffu, suma, off);
        sumb += __shfl_xor_sync(0xffffffffu, sumb, off);
      }
      l_a = l_a * alpha_a + suma;
      l_b = l_b * alpha_b + sumb;
      m_a = mna;
      m_b = mnb;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        oa[e] *= alpha_a;
        ob[e] *= alpha_b;
      }
      // O += P V: lane owns output columns 4 lane .. 4 lane + 3 (16-byte chunk lane / 2, half lane % 2)
      const int j = lane >> 1, region = j >> 3, c = j & 7;
      const uint8_t* vbase = st + C::TILE + region * C::KREG + (lane & 1) * 8;
#pragma unroll 8
      for (int k = 0; k < C::KT; ++k) {
        const float pk_a = __shfl_sync(0xffffffffu, k < 32 ? pa0 : pa1, k & 31);
        const uint2 w = *reinterpret_cast<const uint2*>(vbase + k * 128 + ((c ^ (k & 7)) << 4));
        const float2 v01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
        const float2 v23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
        oa[0] = fmaf(pk_a, v01.x, oa[0]);
        oa[1] = fmaf(pk_a, v01.y, oa[1]);
        oa[2] = fmaf(pk_a, v23.x, oa[2]);
        oa[3] = fmaf(pk_a, v23.y, oa[3]);
        if (vb) {
          const float pk_b = __shfl_sync(0xffffffffu, k < 32 ? pb0 : pb1, k & 31);
          ob[0] = fmaf(pk_b, v01.x, ob[0]);
          ob[1] = fmaf(pk_b, v01.y, ob[1]);
          ob[2] = fmaf(pk_b, v23.x, ob[2]);
          ob[3] = fmaf(pk_b, v23.y, ob[3]);
        }
      }
    }
    __syncthreads();                       // stage t % 2 is free again
    if (tid == 0 && t + 2 < n_tiles) issue(t + 2);
  }
  if (!ok) {
    // let the loads in flight (tiles t_fail and t_fail + 1) land before the CTA exits (bounded)
    if (tid == 0)
      for (int t = t_fail; t < n_tiles && t < t_fail + 2; ++t)
        mbar_wait_quiet(b_full0 + 8 * (t & 1), (t >> 1) & 1, 200000000ull);
    return;
  }
  // the split's normalised partial and its lse
  auto store = [&](int r, float m, float l, const float* o) {
    const int hq = bhq0 + r / a.Lq, i = r % a.Lq;
    const size_t row = (static_cast<size_t>(split) * a.bh + hq) * a.Lq + i;
    const float inv = l > 0.f ? 1.0f / l : 0.f;
    *reinterpret_cast<float4*>(a.part_o + row * D + 4 * lane) = make_float4(o[0] * inv, o[1] * inv, o[2] * inv,
                                                                           o[3] * inv);
    if (lane == 0) a.part_lse[row] = l > 0.f ? (m * c2 + __log2f(l)) * 0.69314718055994531f : -INFINITY;
  };
  if (va) store(ra, m_a, l_a, oa);
  if (vb) store(rb, m_b, l_b, ob);
}

// One warp per query row: lse = ln sum_s e^{lse_s}, O = sum_s e^{lse_s - lse} O_s.
__global__ void fa_decode_merge_kernel(const DecArgs a) {
  constexpr int D = DecCfg::D;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(a.bh) * a.Lq;
  for (long long r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += warps) {
    float mx = -INFINITY;
    for (int s = 0; s < a.n_splits; ++s) mx = fmaxf(mx, a.part_lse[static_cast<size_t>(s) * rows + r]);
    float sum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (mx != -INFINITY) {
      for (int s = 0; s < a.n_splits; ++s) {
        const float ls = a.part_lse[static_cast<size_t>(s) * rows + r];
        if (ls == -INFINITY) continue;
        const float w = __expf(ls - mx);
        sum += w;
        const float4 o = *reinterpret_cast<const float4*>(a.part_o + (static_cast<size_t>(s) * rows + r) * D + 4 * lane);
        acc.x = fmaf(w, o.x, acc.x);
        acc.y = fmaf(w, o.y, acc.y);
        acc.z = fmaf(w, o.z, acc.z);
        acc.w = fmaf(w, o.w, acc.w);
      }
    }
    const float inv = sum > 0.f ? 1.0f / sum : 0.f;
    uint2 out;
    out.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    out.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2*>(a.o + r * D + 4 * lane) = out;
    if (lane == 0) a.lse[r] = sum > 0.f ? mx + __logf(sum) : -INFINITY;
  }
}

}  // namespace fa
