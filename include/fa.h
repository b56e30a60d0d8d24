/*
 * fa.h -- C ABI of the exact IO-aware attention library (libfa.so, sm_100a).
 *
 * What is computed (exact attention, no approximation):
 *     S = scale * Q K^T,  P = softmax_rows(S),  O = P V,
 *     lse_i = ln sum_j exp(S_ij)  (natural log, over unmasked j).
 * Definition: unite.ai, "Flash Attention: Rivoluzionando l'Efficienza dei
 * Modelli Transformer", the standard_attention listing; deepfa.ir, "Flash
 * Attention: بهینه‌سازی مکانیزم توجه در ترنسفورمرها", section on the
 * attention structure.  It is computed tile by tile with the online-softmax
 * rescaling of "La Matematica dietro Flash Attention" (softmax decomposition
 * and merge), so the N x N matrix never reaches device memory.  The backward
 * recomputes P from Q, K and lse (deepfa.ir, section "Technique 2:
 * recomputation") and returns the exact gradients
 *     dV = P^T dO,  dS = P * (dO V^T - D),  D_i = sum_c dO_ic O_ic,
 *     dQ = scale dS K,  dK = scale dS^T Q.
 * Causal masking hides key j from query i when j > i (equal query and key
 * lengths; the general-layout calls below align it bottom-right).
 *
 * Conventions shared by every call:
 *  - Layout of the square calls (fa_fwd, fa_bwd, fa_fwd_ex, the phases,
 *    fa_*_gqa, fa_bwd_noalloc): q, k, v, o, dO, dq, dk, dv are dense row-major
 *    [B, H, N, d] with d innermost (element strides d, N*d, H*N*d); lse is
 *    dense [B, H, N] float.  fa_fwd_general / fa_bwd_general take any lengths,
 *    packed sequences and strides (fa_layout, below).
 *  - All pointers are DEVICE pointers owned by the caller; the library keeps
 *    no reference after the call returns and allocates nothing on these paths.
 *    Every pointer must be non-null and 16-byte aligned.
 *  - Work is enqueued asynchronously on `stream` (0 = legacy default stream);
 *    the functions never synchronise.  Argument errors are reported before
 *    anything is launched.  A kernel whose internal wait gives up (a bug, or a
 *    device that stopped making progress) sets a device status word that
 *    fa_get_device_status() reports; outputs are then undefined.
 *  - Supported: d in {64, 128, 256} for the bf16 forward and backward (head
 *    dimensions up to 256: the nearauto.com FlashAttention-2 digest, section
 *    "新機能: 最大256のヘッドディメンション、マルチクエリアテンション"); the float32
 *    forward (fa_fwd_ex) takes d in {64, 128}; fa_decode takes d in
 *    {64, 128, 256} (the split-key kernel for d == 128); 1 <= N <= 2^24;
 *    B*H*N*d < 2^31 elements per tensor for the square calls.
 *  - scale must be finite and positive (FA_ERR_INVALID otherwise): the
 *    kernels take each row's largest unscaled score as the softmax reference.
 */
#ifndef FA_H
#define FA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID = 1,      /* bad sizes (B, H, N < 1, N too large), scale not finite and > 0,
                              or (device status) inconsistent packed sequence offsets */
  FA_ERR_UNSUPPORTED = 2,  /* d or dtype not supported by this call                 */
  FA_ERR_ALIGN = 3,        /* null or not 16-byte aligned pointer                     */
  FA_ERR_WORKSPACE = 4,    /* workspace missing or smaller than required              */
  FA_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed                    */
  FA_ERR_TIMEOUT = 6       /* a kernel's bounded internal wait gave up                */
} fa_status;

typedef enum {
  FA_BF16 = 0,             /* bfloat16 q, k, v and o                                  */
  FA_F32 = 1               /* float32 q, k, v and o (computed on the bf16 path)       */
} fa_dtype;

/* Opaque CUDA stream handle (a cudaStream_t). */
typedef void* fa_stream_t;

/*
 * Forward, bf16.  q, k, v: [B,H,N,d] bf16 (read); o: [B,H,N,d] bf16 (written);
 * lse: [B,H,N] float (written).  scale multiplies the scores (1/sqrt(d) for the
 * usual attention).  causal != 0 applies the mask j > i.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int N, int d, float scale, int causal, fa_stream_t stream);

/*
 * Forward with an element type.  FA_BF16 behaves like fa_fwd (workspace may be
 * null).  FA_F32: q, k, v, o are float32; q, k, v are first rounded to bf16
 * (nearest-even) into the caller's workspace, the product runs on the bf16
 * tensor-core path with fp32 accumulation, and o is written as float32.
 * workspace: device memory of at least fa_fwd_workspace_size(...) bytes,
 * 256-byte aligned.
 */
fa_status fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                    int B, int H, int N, int d, float scale, int causal, fa_dtype dtype,
                    void* workspace, size_t workspace_bytes, fa_stream_t stream);

/* Bytes of workspace fa_fwd_ex needs (0 for FA_BF16). */
size_t fa_fwd_workspace_size(int B, int H, int N, int d, fa_dtype dtype);

/*
 * Backward, bf16, d in {64, 128, 256}.  Inputs q, k, v, o, dO: [B,H,N,d] bf16; lse from the
 * forward: [B,H,N] float.  Outputs dq, dk, dv: [B,H,N,d] bf16 (written, not
 * accumulated).  workspace: device memory of at least fa_bwd_workspace_size()
 * bytes, 256-byte aligned (holds the fp32 dQ accumulator and per-row D, lse).
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv,
                 int B, int H, int N, int d, float scale, int causal,
                 void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * The three phases fa_bwd runs, in order, on the same stream and workspace;
 * exposed so that callers can schedule (or time) them separately.
 *  fa_bwd_prepare: D_i = sum_c dO_ic O_ic and lse * log2(e) into the
 *                  workspace, and zeroes the fp32 dQ accumulator there.
 *                  Reads o, lse, dout.
 *  fa_bwd_main:    recomputes P and dS from q, k and the prepared rows; writes
 *                  dk, dv (bf16) and adds every dS K contribution into the dQ
 *                  accumulator.  Reads q, k, v, dout.
 *  fa_bwd_finish:  dq = bf16(scale * accumulator).
 * Arguments mean what they mean for fa_bwd.  Calling them out of order, or
 * with different sizes, gives undefined outputs (not a fault).
 */
fa_status fa_bwd_prepare(const void* o, const float* lse, const void* dout, int B, int H, int N, int d,
                         void* workspace, size_t workspace_bytes, fa_stream_t stream);
fa_status fa_bwd_main(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv,
                      int B, int H, int N, int d, float scale, int causal,
                      void* workspace, size_t workspace_bytes, fa_stream_t stream);
fa_status fa_bwd_finish(void* dq, int B, int H, int N, int d, float scale,
                        void* workspace, size_t workspace_bytes, fa_stream_t stream);

/* Bytes of workspace fa_bwd needs. */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Grouped-query (and multi-query) attention: the nearauto.com FlashAttention-2
 * digest, section "新機能: 最大256のヘッドディメンション、マルチクエリアテンション", has a
 * set of query heads share one key/value head (the unite.ai page lists the
 * same variants under "FlashAttention-2").  H query heads, H_kv key/value
 * heads, H a multiple of H_kv; query head h of a batch entry reads key/value
 * head h / (H / H_kv) (contiguous sets).  H_kv == H is fa_fwd / fa_bwd.
 *  q, o, dO, dq: [B,H,N,d] bf16;  k, v, dk, dv: [B,H_kv,N,d] bf16;
 *  lse: [B,H,N] float.  dk and dv of a shared head are the sums over its set.
 * Same layout, ownership, alignment, stream and error rules as fa_fwd /
 * fa_bwd, plus FA_ERR_INVALID when H_kv < 1 or H is not a multiple of H_kv.
 * fa_bwd_gqa takes d in {64, 128, 256} and fa_bwd_workspace_size(B, H, N, d) bytes of
 * workspace (sized by the query heads).
 */
fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse,
                     int B, int H, int H_kv, int N, int d, float scale, int causal, fa_stream_t stream);
fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv,
                     int B, int H, int H_kv, int N, int d, float scale, int causal,
                     void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * General lengths and layouts.  The pages define attention for one square
 * sequence; the integrations they point users to (deepfa.ir, "Flash
 * Attention: بهینه‌سازی مکانیزم توجه در ترنسفورمرها", section on
 * implementation and use: PyTorch, Transformers, vLLM) call it on tensors of
 * other shapes, which these calls accept:
 *  - any number of query rows Nq and key rows Nk (either may be 0);
 *  - fixed lengths (every batch entry has Nq queries and Nk keys) or packed
 *    variable lengths (sequence b is rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]
 *    of the query tensors and cu_seqlens_k[b] .. cu_seqlens_k[b+1] of the
 *    key / value tensors, as in a token-major [total, H, d] batch);
 *  - any element strides for the batch, head and row axes (d contiguous), so
 *    that [B, H, N, d], [B, N, H, d] and views of larger tensors need no copy;
 *  - grouped heads as in fa_fwd_gqa.
 * Causal masking is aligned bottom-right: query i of a sequence with nq
 * queries and nk keys sees keys j <= nk - nq + i (the usual mask when
 * nq == nk).  A query that sees no key (nq > nk under the causal mask, or
 * nk == 0) gets o = 0 and lse = -inf, and contributes no gradient.
 */
typedef struct {
  int64_t batch;   /* elements between batch entries (unused for packed sequences) */
  int64_t head;    /* elements between heads                                    */
  int64_t row;     /* elements between rows (tokens)                            */
} fa_strides;

typedef struct {
  int B;                        /* batch entries (sequences)                                   */
  int H, H_kv;                  /* query heads, key/value heads (H a multiple of H_kv)          */
  int d;                        /* head dim: 64, 128 or 256                                     */
  int Nq, Nk;                   /* fixed lengths: rows per batch entry; packed: an upper bound
                                   on every sequence's length (sets the grid)                   */
  const int32_t* cu_seqlens_q;  /* packed: DEVICE array of B + 1 row offsets; NULL: fixed lengths */
  const int32_t* cu_seqlens_k;  /* packed: likewise for keys and values; NULL with cu_seqlens_q  */
  int total_q, total_k;         /* packed: rows of the query and key tensors (ignored otherwise) */
  fa_strides q, k, v, o;        /* strides of the forward operands                               */
  fa_strides dout, dq, dk, dv;  /* strides of the backward operands (the forward ignores them)   */
} fa_layout;

/*
 * Forward with a general layout (d in {64, 128, 256}).  q, o: [batch][H][row][d] bf16 with strides
 * layout->q, layout->o; k, v: [batch][H_kv][row][d] bf16.  lse (float, dense):
 * [B, H, Nq] for fixed lengths, [H, total_q] for packed sequences.  Strides
 * of axes longer than 1 must be positive multiples of 8 elements (16 bytes)
 * (FA_ERR_ALIGN); every pointer non-null and 16-byte aligned.  Nq == 0 (or
 * total_q == 0) launches nothing.  Packed offsets are read on the device: a
 * sequence whose offsets are out of order, outside the tensors or longer
 * than Nq / Nk is skipped (nothing written for it) and fa_get_device_status()
 * then reports FA_ERR_INVALID.  Same ownership, stream and error rules as
 * fa_fwd otherwise; `layout` is read during the call only.
 */
fa_status fa_fwd_general(const void* q, const void* k, const void* v, void* o, float* lse,
                         const fa_layout* layout, float scale, int causal, fa_stream_t stream);

/*
 * Backward with a general layout (d in {64, 128, 256}): the exact gradients of fa_fwd_general.
 * Inputs q, k, v, o, dout (strides layout->q, k, v, o, dout) and lse from the
 * forward (its layout); outputs dq, dk, dv (strides layout->dq, dk, dv),
 * written, not accumulated; dk and dv of a shared head sum over its set.
 * workspace: at least fa_bwd_general_workspace_size(layout) bytes, 256-byte
 * aligned.  Same rules as fa_fwd_general and fa_bwd otherwise.
 */
fa_status fa_bwd_general(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv, const fa_layout* layout,
                         float scale, int causal, void* workspace, size_t workspace_bytes,
                         fa_stream_t stream);

/* Bytes of workspace fa_bwd_general needs (0 for a layout it rejects). */
size_t fa_bwd_general_workspace_size(const fa_layout* layout);

/*
 * Decoding: Lq queries that are the last Lq positions of a sequence of Nk keys
 * (a key/value cache), with the keys split across CTAs and the partial results
 * combined by the softmax merge of the unite.ai page "Flash Attention:
 * Rivoluzionando l'Efficienza dei Modelli Transformer", section "La Matematica
 * dietro Flash Attention".  The decode workload is the one the gist.science
 * FlashAttention-V page times.
 *  q, o: [B,H,Lq,d] bf16;  k, v: [B,H_kv,Nk,d] bf16 (H a multiple of H_kv, as
 *  in fa_fwd_gqa);  lse: [B,H,Lq] float (natural log).
 *  causal != 0: query i sees keys j <= Nk - Lq + i (bottom-right alignment).
 * d in {64, 128, 256} (FA_ERR_UNSUPPORTED otherwise), 1 <= Lq <= Nk and
 * B * H_kv <= 65535 (FA_ERR_INVALID).  workspace: at least
 * fa_decode_workspace_size(...) bytes, 256-byte aligned (the per-split partial
 * outputs); same layout, ownership, alignment, stream and error rules as
 * fa_fwd otherwise.  With d == 128 and (H / H_kv) * Lq <= 16 two kernels run:
 * the split partials, then the merge; other shapes run the general forward
 * (fa_fwd_general with N_q = Lq), which computes the same result.
 */
fa_status fa_decode(const void* q, const void* k, const void* v, void* o, float* lse,
                    int B, int H, int H_kv, int Lq, int Nk, int d, float scale, int causal,
                    void* workspace, size_t workspace_bytes, fa_stream_t stream);

/* Bytes of workspace fa_decode needs (0 for invalid sizes). */
size_t fa_decode_workspace_size(int B, int H, int H_kv, int Lq, int Nk, int d);

/*
 * Backward without a caller-supplied workspace.  Same arguments, outputs and
 * numerics as fa_bwd, minus the workspace pair.  The pages have no counterpart
 * of this call; it exists for callers that cannot allocate device memory
 * themselves -- for example a plug-in whose host application owns every
 * device allocation through its own pool, or a serving path that must not
 * allocate once it has started -- and so cannot hand fa_bwd a workspace.
 *
 * The scratch lives in one statically sized device array inside libfa.so
 * (FA_NOALLOC_SCRATCH_BYTES bytes, held on every GPU that loads the library
 * until the process exits).  Shapes whose fa_bwd_workspace_size() exceeds it
 * are rejected with FA_ERR_WORKSPACE before anything is launched.  This call
 * never allocates (no cudaMalloc, no allocating library routine).
 *
 * The first call on a device (with that device current) looks up the array's
 * device address; make that first call before any stream capture.  After a
 * device reset the next call looks it up again (it is tied to the context).  All calls
 * on a device share the one array and leave their contents in it: the dQ
 * accumulator is cleared on every call, but two calls that overlap on the GPU
 * (different streams, no ordering between them) race and give wrong results.
 */
#define FA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv,
                         int B, int H, int N, int d, float scale, int causal, fa_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the device status word of the
 * current device.  Returns FA_ERR_TIMEOUT if any kernel since the last call
 * gave up a bounded wait, FA_ERR_CUDA if the synchronisation failed or a
 * kernel found its shared-memory allocation too small for its buffers (it then
 * did no work), FA_ERR_INVALID if a kernel found inconsistent packed sequence
 * offsets (it skipped those sequences), else FA_OK.
 */
fa_status fa_get_device_status(fa_stream_t stream);

/*
 * Diagnostic: launches one tiny kernel that waits on a shared-memory barrier
 * nothing will ever complete, bounded by timeout_ns (clamped to [1 ms, 2 s]).
 * The kernel gives up, sets the status word and returns; the caller then sees
 * FA_ERR_TIMEOUT from fa_get_device_status().  Used to test that path.
 */
fa_status fa_selftest_wait_timeout(uint64_t timeout_ns, fa_stream_t stream);

/* Human-readable name of a status code. */
const char* fa_status_string(fa_status s);

/* Library version, e.g. "0.1.0". */
const char* fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H */
