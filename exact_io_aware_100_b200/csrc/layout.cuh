// Where the rows of each sequence live, shared by the forward and backward
// kernels.
//
// Two batch layouts:
//  * fixed lengths: batch entry b has Nq query rows and Nk key rows; a tensor
//    is [batch][head][row][d] with any element strides (d contiguous), so
//    [B, H, N, d] and [B, N, H, d] are both covered;
//  * variable lengths: sequence b is the packed rows cu_q[b]..cu_q[b+1] of
//    the queries (cu_k for keys and values) of tensors [rows][head][d] (again
//    with any row and head strides); Nq and Nk are then the longest sequence.
// The causal mask is aligned bottom-right: query i of a sequence with nq
// queries and nk keys sees keys j <= nk - nq + i (the usual mask when
// nq == nk); a query that sees no key gets O = 0 and lse = -inf.
#pragma once

#include "ptx.cuh"

namespace fa {

struct Strides {   // element strides of a [batch][head][row][d] operand
  long long b, h, r;
};

struct SeqLayout {
  const int* cu_q;     // variable lengths: B + 1 query row offsets (device); null for fixed lengths
  const int* cu_k;     // likewise for keys and values
  int B, H, H_kv;
  int Nq, Nk;          // rows per sequence (fixed), or the longest sequence (variable)
  int total_q, total_k;  // variable lengths: rows of the packed tensors
};

struct SeqSpan {
  int q0, nq;          // first query row coordinate, query rows
  int k0, nk;          // first key row coordinate, key rows
  int bc;              // batch coordinate (0 for packed sequences)
};

// Rows of sequence b.  PACKED reads the offsets (variable lengths); otherwise
// everything comes from the kernel parameters, which keeps it out of registers.
// Offsets that are out of order, outside the packed tensors or longer than the
// stated maximum flag DEV_ARGS and give an empty sequence, so nothing is read
// or written for it.
template <bool PACKED>
__device__ __forceinline__ SeqSpan seq_span(const SeqLayout& L, int b, uint32_t* status) {
  SeqSpan s;
  if constexpr (!PACKED) {
    s.q0 = 0;
    s.nq = L.Nq;
    s.k0 = 0;
    s.nk = L.Nk;
    s.bc = b;
    return s;
  } else {
    const int qa = __ldg(L.cu_q + b), qe = __ldg(L.cu_q + b + 1);
    const int ka = __ldg(L.cu_k + b), ke = __ldg(L.cu_k + b + 1);
    const bool ok = 0 <= qa && qa <= qe && qe <= L.total_q && qe - qa <= L.Nq && 0 <= ka && ka <= ke &&
                    ke <= L.total_k && ke - ka <= L.Nk;
    if (!ok) {
      atomicOr(status, DEV_ARGS);
      s.q0 = s.nq = s.k0 = s.nk = s.bc = 0;
      return s;
    }
    s.q0 = qa;
    s.nq = qe - qa;
    s.k0 = ka;
    s.nk = ke - ka;
    s.bc = 0;
    return s;
  }
}

__device__ __forceinline__ SeqSpan seq_span_any(const SeqLayout& L, int b, uint32_t* status) {
  return L.cu_q ? seq_span<true>(L, b, status) : seq_span<false>(L, b, status);
}

// Index of query row r of sequence s, head h, in the per-row vectors (lse) and
// in the fp32 dQ accumulator (times d): [B][H][Nq] for fixed lengths,
// [H][total_q] for packed sequences.
template <bool PACKED>
__device__ __forceinline__ long long row_index(const SeqLayout& L, const SeqSpan& s, int h, int r) {
  if constexpr (PACKED) return static_cast<long long>(h) * L.total_q + s.q0 + r;
  else return (static_cast<long long>(s.bc) * L.H + h) * L.Nq + r;
}

__device__ __forceinline__ long long row_index_any(const SeqLayout& L, const SeqSpan& s, int h, int r) {
  return L.cu_q ? row_index<true>(L, s, h, r) : row_index<false>(L, s, h, r);
}

// Element offset of row `row` (a row coordinate: s.q0 / s.k0 already added)
// of head h in an operand with strides st.
__device__ __forceinline__ long long row_offset(const Strides& st, int bc, int h, int row) {
  return bc * st.b + h * st.h + static_cast<long long>(row) * st.r;
}

}  // namespace fa
