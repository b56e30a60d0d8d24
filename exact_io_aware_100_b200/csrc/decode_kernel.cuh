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
//    (at most 16 rows).  64-key tiles of K and V stream through a three-stage
//    TMA ring (128-byte swizzle, so per-lane shared reads are conflict free);
//    three block barriers per tile: the one that opens a tile also releases
//    the previous tile's stage and score rows (its TMA reload is issued
//    right after it).
//    Per tile, every warp works whatever the row count: scores with four
//    adjacent lanes per key (a quarter of d each, all rows, packed fp32x2
//    FMAs, summed by two shuffles; each K element is read from shared memory
//    once), the online softmax with one warp per row, and P.V with each warp
//    taking 8 of the 64 keys for all rows (four output columns per lane),
//    keeping a partial O over its keys that the warps sum once at the end of
//    the split.  Decoding is bound by HBM, so the kernel is built to spend as
//    few issue slots per byte as it can.  Writes the split's normalised partial O
//    (fp32) and its lse (-inf when no key is visible);
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
  // fp32 query rows, each d-quarter padded by 16 B so the four quarters a warp
  // reads at once sit in different banks; reused as [R_MAX][D] to sum the
  // warps' partial O at the end
  static constexpr int Q_QUARTER = 36;           // floats per d-quarter (32 + 4 padding)
  static constexpr int Q_ROW = 4 * Q_QUARTER;    // floats per query row
  static constexpr int OFF_Q = 0;
  static constexpr int STAGES = 3;
  static constexpr int OFF_ST = R_MAX * Q_ROW * 4;   // STAGES stages of K then V (1 KB aligned)
  static constexpr int STAGE = 2 * TILE;
  static constexpr int OFF_S = OFF_ST + STAGES * STAGE;     // fp32 [R_MAX][KT]: scores, then P
  static constexpr int OFF_ROW = OFF_S + R_MAX * KT * 4;    // fp32 [R_MAX]: alpha of the tile, then l
  static constexpr int OFF_BAR = OFF_ROW + R_MAX * 4;
  static constexpr int OFF_MISC = OFF_BAR + 8 * STAGES;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;   // + alignment slack
};

// Splits for a cache of Nk keys and bh_kv key/value heads: about 1152 CTAs in
// total (several waves at two CTAs per SM), each split a whole number of 64-key
// tiles.  Against 768, 1024 and 2048 CTAs, 1152 measured 2-5 % faster on
// 8192- to 65536-key caches with 32 to 512 key/value heads.
__host__ __device__ inline int decode_splits(int bh_kv, int Nk, int* split_keys) {
  const int tiles = (Nk + DecCfg::KT - 1) / DecCfg::KT;
  int want = (1152 + bh_kv - 1) / bh_kv;
  if (want < 1) want = 1;
  if (want > tiles) want = tiles;
  const int tiles_per = (tiles + want - 1) / want;
  *split_keys = tiles_per * DecCfg::KT;
  return (tiles + tiles_per - 1) / tiles_per;
}

// RM: a bound on the rows (4, 8 or 16), which sizes the partial-O registers.
template <int RM>
__global__ void __launch_bounds__(DecCfg::THREADS, 2)
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
    for (int st = 0; st < C::STAGES; ++st) mbar_init(b_full0 + 8 * st, 1);
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
    sq[r * C::Q_ROW + (c >> 5) * C::Q_QUARTER + (c & 31)] = x;
  }
  __syncthreads();
  const WaitCtl ctl{abort_flag, a.status, a.wait_limit_ns};
  auto issue = [&](int t) {         // tile t of this split into stage t % STAGES (thread 0)
    const uint32_t st = sbase + C::OFF_ST + (t % C::STAGES) * C::STAGE;
    const uint32_t bar = b_full0 + 8 * (t % C::STAGES);
    mbar_expect_tx(bar, 2 * C::TILE);
    const int y = k_begin + t * C::KT;
    for (int r = 0; r < 2; ++r) {
      tma_load_3d(st + r * C::KREG, &tm_k, bar, r * 64, y, bhkv);
      tma_load_3d(st + C::TILE + r * C::KREG, &tm_v, bar, r * 64, y, bhkv);
    }
  };
  if (tid == 0) {
    for (int t = 0; t < C::STAGES && t < n_tiles; ++t) issue(t);
  }

  float* ss = reinterpret_cast<float*>(smem + C::OFF_S);     // [R_MAX][KT]
  float* srow = reinterpret_cast<float*>(smem + C::OFF_ROW); // [R_MAX]
  const float c2 = a.scale_log2;
  // causal limit of row r: key positions <= lim are visible
  auto lim_of = [&](int r) { return a.causal ? a.Nk - a.Lq + r % a.Lq : a.Nk - 1; };
  // scores: thread = (key sk, quarter dq of d), lanes 4 sk .. 4 sk + 3 of a warp hold one key
  const int sk = tid >> 2, dq = tid & 3;
  // softmax: warp w owns rows w and w + 8 (running max m and sum l)
  const int ra = warp, rb = warp + 8;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
  // P.V: warp w takes keys 8w .. 8w + 7 of every tile; lane owns columns 4 lane .. 4 lane + 3
  float2 acc01[RM], acc23[RM];          // columns 4 lane, 4 lane + 1 and 4 lane + 2, 4 lane + 3
#pragma unroll
  for (int r = 0; r < RM; ++r) acc01[r] = acc23[r] = make_float2(0.f, 0.f);
  const int pj = lane >> 1, pregion = pj >> 3, pc = pj & 7;
  bool ok = true;
  int t_fail = n_tiles;
  for (int t = 0; t < n_tiles; ++t) {
    ok = ok && mbar_wait(b_full0 + 8 * (t % C::STAGES), (t / C::STAGES) & 1, ctl);
    if (!__syncthreads_and(ok)) { ok = false; t_fail = t; break; }   // every thread agrees before using the stage
    // every thread is past tile t-1's P.V: its stage can be reloaded, its score rows rewritten
    if (tid == 0 && t >= 1 && t - 1 + C::STAGES < n_tiles) issue(t - 1 + C::STAGES);
    const uint8_t* st = smem + C::OFF_ST + (t % C::STAGES) * C::STAGE;
    const int kt0 = k_begin + t * C::KT;
    // ---- scores S[r][sk]: this lane's quarter of d for every row, then the quarters summed
    {
      const uint8_t* krow = st + (dq >> 1) * C::KREG + sk * 128;
      float2 kf[16];                       // d = 32 dq + 2 m, 32 dq + 2 m + 1
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 w = *reinterpret_cast<const uint4*>(krow + ((((dq & 1) * 4 + i) ^ (sk & 7)) << 4));
        kf[4 * i + 0] = bf16x2_to_float2(w.x);
        kf[4 * i + 1] = bf16x2_to_float2(w.y);
        kf[4 * i + 2] = bf16x2_to_float2(w.z);
        kf[4 * i + 3] = bf16x2_to_float2(w.w);
      }
      const int pos = kt0 + sk;
#pragma unroll
      for (int r = 0; r < RM; ++r) {
        if (r < R) {                       // uniform across the CTA
          const float4* qp = reinterpret_cast<const float4*>(sq + r * C::Q_ROW + dq * C::Q_QUARTER);
          float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 qa = qp[2 * i], qb = qp[2 * i + 1];
            a0 = ffma2(make_float2(qa.x, qa.y), kf[4 * i + 0], a0);
            a1 = ffma2(make_float2(qa.z, qa.w), kf[4 * i + 1], a1);
            a0 = ffma2(make_float2(qb.x, qb.y), kf[4 * i + 2], a0);
            a1 = ffma2(make_float2(qb.z, qb.w), kf[4 * i + 3], a1);
          }
          float x = (a0.x + a0.y) + (a1.x + a1.y);
          x += __shfl_xor_sync(0xffffffffu, x, 1);
          x += __shfl_xor_sync(0xffffffffu, x, 2);
          if (dq == 0) ss[r * C::KT + sk] = (pos < k_end && pos <= lim_of(r)) ? x : -INFINITY;
        }
      }
    }
    __syncthreads();
    // ---- online softmax: rows ra and rb of this warp; P back into ss, the tile's alpha into srow
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = h ? rb : ra;
      if (r < R) {
        float& m = h ? m_b : m_a;
        float& l = h ? l_b : l_a;
        const float s0 = ss[r * C::KT + lane], s1 = ss[r * C::KT + lane + 32];
        float mt = fmaxf(s0, s1);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
        const float mn = fmaxf(m, mt);
        // a row that has seen no visible key keeps m = -inf and contributes nothing
        const float alpha = (mn == -INFINITY) ? 1.f : ex2_approx((m - mn) * c2);
        const float nb = (mn == -INFINITY) ? 0.f : mn * c2;
        const float p0 = ex2_approx(fmaf(s0, c2, -nb)), p1 = ex2_approx(fmaf(s1, c2, -nb));
        float sum = p0 + p1;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        l = l * alpha + sum;
        m = mn;
        ss[r * C::KT + lane] = p0;
        ss[r * C::KT + lane + 32] = p1;
        if (lane == 0) srow[r] = alpha;
      }
    }
    __syncthreads();
    // ---- P.V over this warp's 8 keys, for every row
    const uint8_t* vbase = st + C::TILE + pregion * C::KREG + (lane & 1) * 8;
#pragma unroll
    for (int r = 0; r < RM; ++r) {
      if (r < R) {
        const float al = srow[r];
        acc01[r] = fmul2(acc01[r], make_float2(al, al));
        acc23[r] = fmul2(acc23[r], make_float2(al, al));
      }
    }
#pragma unroll
    for (int half = 0; half < 2; ++half) {   // keys 8 warp + 4 half .. + 3
      float2 v01[4], v23[4];
#pragma unroll
      for (int kq = 0; kq < 4; ++kq) {
        const int k = 8 * warp + 4 * half + kq;
        const uint2 w = *reinterpret_cast<const uint2*>(vbase + k * 128 + ((pc ^ (k & 7)) << 4));
        v01[kq] = bf16x2_to_float2(w.x);
        v23[kq] = bf16x2_to_float2(w.y);
      }
#pragma unroll
      for (int r = 0; r < RM; ++r) {
        if (r < R) {
          const float4 p = *reinterpret_cast<const float4*>(ss + r * C::KT + 8 * warp + 4 * half);
          acc01[r] = ffma2(make_float2(p.x, p.x), v01[0], acc01[r]);
          acc23[r] = ffma2(make_float2(p.x, p.x), v23[0], acc23[r]);
          acc01[r] = ffma2(make_float2(p.y, p.y), v01[1], acc01[r]);
          acc23[r] = ffma2(make_float2(p.y, p.y), v23[1], acc23[r]);
          acc01[r] = ffma2(make_float2(p.z, p.z), v01[2], acc01[r]);
          acc23[r] = ffma2(make_float2(p.z, p.z), v23[2], acc23[r]);
          acc01[r] = ffma2(make_float2(p.w, p.w), v01[3], acc01[r]);
          acc23[r] = ffma2(make_float2(p.w, p.w), v23[3], acc23[r]);
        }
      }
    }
  }
  if (!ok) {
    // let the loads in flight land before the CTA exits (bounded): tiles t_fail .. last issued
    const int last_issued = C::STAGES - 1 + (t_fail > 1 ? t_fail - 1 : 0);
    if (tid == 0)
      for (int t = t_fail; t < n_tiles && t <= last_issued; ++t)
        mbar_wait_quiet(b_full0 + 8 * (t % C::STAGES), (t / C::STAGES) & 1, 200000000ull);
    return;
  }
  __syncthreads();                         // every warp is done with the last tile's P and alphas
  // ---- sum the warps' partial O (in the query buffer, which is no longer needed), then normalise
  for (int idx = tid; idx < C::R_MAX * D; idx += C::THREADS) sq[idx] = 0.f;
  if (lane == 0) {
    if (ra < R) srow[ra] = l_a;
    if (rb < R) srow[rb] = l_b;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < RM; ++r) {
    if (r < R) {
      atomicAdd(sq + r * D + 4 * lane + 0, acc01[r].x);
      atomicAdd(sq + r * D + 4 * lane + 1, acc01[r].y);
      atomicAdd(sq + r * D + 4 * lane + 2, acc23[r].x);
      atomicAdd(sq + r * D + 4 * lane + 3, acc23[r].y);
    }
  }
  __syncthreads();
  // thread = (row, 16-byte group of columns) writes the split's normalised partial
  for (int idx = tid; idx < R * (D / 4); idx += C::THREADS) {
    const int r = idx / (D / 4), c4 = idx % (D / 4);
    const int hq = bhq0 + r / a.Lq, i = r % a.Lq;
    const size_t row = (static_cast<size_t>(split) * a.bh + hq) * a.Lq + i;
    const float l = srow[r];
    const float inv = l > 0.f ? 1.0f / l : 0.f;
    const float4 v = *reinterpret_cast<const float4*>(sq + r * D + 4 * c4);
    *reinterpret_cast<float4*>(a.part_o + row * D + 4 * c4) = make_float4(v.x * inv, v.y * inv, v.z * inv, v.w * inv);
  }
  if (lane == 0) {
    auto put_lse = [&](int r, float m, float l) {
      const int hq = bhq0 + r / a.Lq, i = r % a.Lq;
      const size_t row = (static_cast<size_t>(split) * a.bh + hq) * a.Lq + i;
      a.part_lse[row] = l > 0.f ? (m * c2 + __log2f(l)) * 0.69314718055994531f : -INFINITY;
    };
    if (ra < R) put_lse(ra, m_a, l_a);
    if (rb < R) put_lse(rb, m_b, l_b);
  }
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
