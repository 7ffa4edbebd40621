/*
 * kvc.h — C ABI of the B200 (sm_100a) token-level KV compressor.
 *
 * The compressor turns every m consecutive tokens of a sequence into one compressed
 * KV entry by a per-channel softmax-weighted pool.  Sources (web pages):
 *   [SC]  "序列压缩注意力" (sequence-compressed attention):
 *         eq. attn-seqcomp-csa-proj     C^a = H W^{KV_a}, C^b = H W^{KV_b}, Z^a = H W^{Z_a}, Z^b = H W^{Z_b}
 *         eq. attn-seqcomp-csa-softmax  [S^a; S^b] = Softmax_row([Z^a_{mi..m(i+1)-1} + B^a; Z^b_{m(i-1)..mi-1} + B^b])
 *         eq. attn-seqcomp-csa-pool     C^Comp_i = sum_j S^a_j (.) C^a_j + sum_j S^b_j (.) C^b_j
 *         table attn-seqcomp-overlap    a-range(i) = [mi, m(i+1)-1], b-range(i) = [m(i-1), mi-1]
 *         eq. attn-seqcomp-overlap-bound  Z^b_{-m:-1} = -inf, C^b_{-m:-1} = 0 (entry 0)
 *         eq. attn-seqcomp-hca          S = Softmax_row(Z + B), C^Comp_i = sum_{j in segment i} S_j (.) C_j, m' = 128
 *   [CSA] "Ch 04 · CSA" (DeepSeek-V4 book), §3 Token-Level Compressor (same equations, 12-token example).
 *   [HCA] "Ch 05 · HCA" (DeepSeek-V4 book), §2 compression formulas.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.  All tensors are dense, row-major, channel fastest:
 *   streams  [batch, n, c]   (sequence b, token t, channel ch at ((b*n)+t)*c+ch)
 *   biases   [m, c] fp32     (row k = in-block position k)
 *   H        [batch*n, d]    bf16 (sequence b = rows b*n .. b*n+n-1)
 *   W        [d, c]          bf16 (as in C = H W)
 *   out      [batch, N_e, c] with N_e = floor(n/m) = kvc_num_entries(n, m).
 * Entries.  Sequence b's entry i reads only tokens of sequence b.  The trailing n mod m
 *   tokens of a sequence form no complete block and are not compressed.
 * Ownership.  Every tensor pointer is a DEVICE pointer on the current CUDA device,
 *   owned by the caller.  The library never allocates, frees or retains them.
 * Asynchrony.  Work is enqueued on `stream` (NULL = the legacy default stream) and the
 *   call returns after the enqueue; no implicit synchronisation, no host<->device copy.
 * Arithmetic.  Inputs are widened to fp32; logits, softmax and the weighted sum are
 *   fp32 (the fused path accumulates H W in fp32 on the tensor cores and never rounds
 *   the streams); bf16 outputs are rounded to nearest even.
 * Errors.  Arguments are validated on the host before any launch; on error nothing is
 *   enqueued and the status says why:
 *     KVC_ERR_NULL         a required pointer is NULL
 *     KVC_ERR_SHAPE        negative size, c not a multiple of 8, m < 1, overlap not 0/1,
 *                          size overflow, fused d % 64 != 0 or c % 128 != 0
 *     KVC_ERR_DTYPE        unknown dtype or unsupported dtype combination
 *     KVC_ERR_ALIGN        a stream, H, W or out pointer is not 16-byte aligned, or a
 *                          bias pointer is not 4-byte aligned
 *     KVC_ERR_UNSUPPORTED  valid but outside what the kernels implement (e.g. window too long)
 *     KVC_ERR_CUDA         the launch (or a CUDA query it needs) failed
 *     KVC_ERR_TIMEOUT      reported by kvc_device_status(): a bounded wait inside a
 *                          kernel gave up (the kernel then skipped its remaining work)
 *     KVC_ERR_POINTER      a tensor pointer is not device (or managed) memory of the
 *                          current device (e.g. a host pointer)
 *     KVC_ERR_INDEX        reported by kvc_device_status(): an entry list read from device
 *                          memory named a window outside its sequence or the streams (that
 *                          entry was skipped and its output row left unwritten)
 *     KVC_ERR_TOO_LARGE    hca_compress_noalloc: the bias needs more than its fixed scratch
 *     KVC_ERR_WORKSPACE    reported by kvc_device_status(): hca_compress_prepared was given
 *                          a workspace that hca_prepare_bias did not fill for the same c, m
 *                          and stream dtype (nothing was computed)
 *   An empty problem (batch == 0 or N_e == 0) is valid: KVC_OK, nothing is launched and
 *   no pointer is dereferenced.
 * Thread safety.  Calls may be made concurrently from several host threads.  A kernel's
 *   dynamic shared-memory limit is raised once to the device's maximum (under a lock)
 *   and never lowered, so concurrent calls with different window lengths do not
 *   interfere.  The device error words read by kvc_device_status() are per device.
 */
#ifndef KVC_H
#define KVC_H

#include <stdint.h>

#if defined(__GNUC__)
#define KVC_API __attribute__((visibility("default")))
#else
#define KVC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kvc_status {
  KVC_OK = 0,
  KVC_ERR_NULL = 1,
  KVC_ERR_SHAPE = 2,
  KVC_ERR_DTYPE = 3,
  KVC_ERR_ALIGN = 4,
  KVC_ERR_UNSUPPORTED = 5,
  KVC_ERR_CUDA = 6,
  KVC_ERR_TIMEOUT = 7,
  KVC_ERR_POINTER = 8,
  KVC_ERR_INDEX = 9,
  KVC_ERR_WORKSPACE = 10,
  KVC_ERR_TOO_LARGE = 11
} kvc_status;

typedef enum kvc_dtype { KVC_F32 = 0, KVC_BF16 = 1 } kvc_dtype;

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st* kvc_stream;

/* Number of compressed entries of an n-token sequence at ratio m: floor(n / m)
 * ([CSA] §3 cuts the sequence into floor(n/m) segments; [SC] table
 * attn-seqcomp-csa-hca: ~n/m entries).  Returns -1 if n < 0 or m < 1. */
KVC_API int64_t kvc_num_entries(int64_t n, int32_t m);

/* Human-readable name of a status code (static storage, never NULL). */
KVC_API const char* kvc_status_string(kvc_status s);

/* CSA compressor over precomputed streams ([SC] eqs. attn-seqcomp-csa-softmax,
 * attn-seqcomp-csa-pool, attn-seqcomp-overlap-bound; [CSA] §3).
 *   Ca, Cb, Za, Zb : streams [batch, n, c], dtype in_dtype (KVC_F32 or KVC_BF16)
 *   Ba, Bb         : position biases [m, c] fp32
 *   overlap = 1    : entry i pools the 2m rows a-range(i) of (Ca, Za + Ba) and
 *                    b-range(i) of (Cb, Zb + Bb) under one joint per-channel softmax;
 *                    entry 0 has no b-rows (logit -inf, vector 0).
 *   overlap = 0    : entry i pools its own m rows of (Ca, Za + Ba) only; Cb, Zb and Bb
 *                    are not read and may be NULL.
 *   out            : [batch, N_e, c], dtype out_dtype (KVC_F32 or KVC_BF16). */
KVC_API kvc_status csa_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                        kvc_dtype in_dtype, const float* Ba, const float* Bb,
                        int64_t batch, int64_t n, int64_t c, int32_t m, int32_t overlap,
                        void* out, kvc_dtype out_dtype, kvc_stream stream);

/* HCA compressor ([SC] eq. attn-seqcomp-hca; [HCA] §2): entry i pools the m rows
 * [m i, m(i+1)-1] of C under Softmax_row(Z + B), no overlap, single stream.
 *   C, Z : [batch, n, c] in_dtype;  B : [m, c] fp32;  out : [batch, N_e, c] out_dtype.
 *   m is the compression ratio m' (128 on the pages); windows of up to 320 rows are
 *   supported (KVC_ERR_UNSUPPORTED beyond). */
KVC_API kvc_status hca_compress(const void* C, const void* Z, kvc_dtype in_dtype, const float* B,
                        int64_t batch, int64_t n, int64_t c, int32_t m,
                        void* out, kvc_dtype out_dtype, kvc_stream stream);

/* Prepared position bias for the HCA compressor.  The bias B [m, c] is a learned weight,
 * the same in every call, while every call of hca_compress stages it afresh in each CTA
 * (scaled by log2 e, reordered for the consumers, per-channel maxima and spread for the
 * softmax reference); on short sequences that staging is a sizeable part of the call.
 * hca_prepare_bias does it once into a caller-owned device workspace, which
 * hca_compress_prepared then copies into shared memory as it stands.  The result is bit
 * for bit that of hca_compress with the same B.
 *   hca_bias_workspace_bytes: the workspace size for (c, m, in_dtype) (the stream dtype the
 *     workspace will serve); -1 for invalid arguments.
 *   hca_prepare_bias: B [m, c] fp32 device (4-byte aligned) -> workspace (device, 256-byte
 *     aligned, at least hca_bias_workspace_bytes); c % 8 == 0, 1 <= m <= 320.  Asynchronous
 *     on `stream`; the workspace holds no pointer to B, which may change afterwards.
 *   hca_compress_prepared: as hca_compress with B replaced by a workspace that
 *     hca_prepare_bias filled for the same c, m and in_dtype (checked on the device: a
 *     mismatch computes nothing and kvc_device_status() reports KVC_ERR_WORKSPACE).  The
 *     workspace is only read; calls may share it. */
KVC_API int64_t hca_bias_workspace_bytes(int64_t c, int32_t m, kvc_dtype in_dtype);
KVC_API kvc_status hca_prepare_bias(const float* B, int64_t c, int32_t m, kvc_dtype in_dtype,
                                    void* workspace, int64_t workspace_bytes, kvc_stream stream);
KVC_API kvc_status hca_compress_prepared(const void* C, const void* Z, kvc_dtype in_dtype,
                                         const void* workspace, int64_t workspace_bytes,
                                         int64_t batch, int64_t n, int64_t c, int32_t m,
                                         void* out, kvc_dtype out_dtype, kvc_stream stream);

/* hca_compress without any memory of the caller's beyond inputs and outputs, and without
 * allocating any (no cudaMalloc, cudaFree or allocating library call).  This entry point
 * has no counterpart in the pages: it serves callers that cannot allocate device memory
 * while they run, e.g. a serving loop whose device memory is all handed out at start-up
 * (a later cudaMalloc can fail, and can synchronise the device), or a host program with no
 * allocator of its own to provide the workspace of hca_prepare_bias.
 *   Arguments and result as hca_compress.  Each call prepares the bias (as hca_prepare_bias
 *   does) into a fixed scratch array inside the library, then runs hca_compress_prepared on
 *   it; the result is bit for bit hca_compress's.
 *   Scratch: one 1 MiB array in device memory per device that loads the library, held until
 *   the process exits.  A call whose workspace (hca_bias_workspace_bytes(c, m, in_dtype))
 *   exceeds 1 MiB returns KVC_ERR_TOO_LARGE before any launch: about 8 m c bytes, e.g. c up
 *   to 1008 at m = 128.
 *   Set-up: the first call on a device that launches work looks up the array's device
 *   address (cudaGetSymbolAddress, which may load the library's device code) and keeps it
 *   for later calls on that device; make that first call before any stream capture, and
 *   call it no more on a device after cudaDeviceReset there.
 *   Every call shares the scratch and leaves its contents behind; each call rewrites all it
 *   reads before reading it, so nothing needs clearing.  Calls whose work may overlap on
 *   the GPU (other streams, other host threads) race on the scratch: issue them in order on
 *   one stream, or synchronise between them. */
KVC_API kvc_status hca_compress_noalloc(const void* C, const void* Z, kvc_dtype in_dtype,
                                        const float* B, int64_t batch, int64_t n, int64_t c,
                                        int32_t m, void* out, kvc_dtype out_dtype,
                                        kvc_stream stream);

/* Scalar-logit CSA compressor ([CSA] §3 symbol table: one score per token and stream,
 * an m-dimensional position bias, and a scalar weight S_j on the whole vector C_j).
 *   Ca, Cb : [batch, n, c] in_dtype (16-byte aligned);  za, zb : [batch, n] in_dtype
 *   (element aligned);  ba, bb : [m] fp32;  out : [batch, N_e, c] out_dtype.
 *   Entry i: w = softmax over the 2m scalars [za[mi..m(i+1)-1] + ba ; zb[m(i-1)..mi-1] + bb]
 *   (entry 0: its m a-rows only), C^Comp_i = sum_j w_j C_j, the same w for every
 *   channel.  overlap = 0: a-rows only; Cb, zb and bb are not read and may be NULL.
 *   Windows of up to 320 rows. */
KVC_API kvc_status csa_compress_scalar_logits(const void* Ca, const void* Cb, const void* za,
                                              const void* zb, kvc_dtype in_dtype,
                                              const float* ba, const float* bb, int64_t batch,
                                              int64_t n, int64_t c, int32_t m, int32_t overlap,
                                              void* out, kvc_dtype out_dtype, kvc_stream stream);

/* Scalar-logit HCA compressor ([HCA] §2 with an m'-dimensional bias): entry i pools the
 * m rows of segment i of C with w = softmax(z[mi..m(i+1)-1] + b).
 *   C : [batch, n, c] in_dtype;  z : [batch, n] in_dtype;  b : [m] fp32. */
KVC_API kvc_status hca_compress_scalar_logits(const void* C, const void* z, kvc_dtype in_dtype,
                                              const float* b, int64_t batch, int64_t n,
                                              int64_t c, int32_t m, void* out,
                                              kvc_dtype out_dtype, kvc_stream stream);

/* Entry lists: the CSA compressor for an arbitrary set of entries of sequences packed
 * one after another in the streams (decode: each sequence that just completed a block
 * emits its new entry; ragged prefill: every entry of sequences of different lengths).
 *   Ca, Cb, Za, Zb : packed streams [total_rows, c] in_dtype;  Ba, Bb : [m, c] fp32
 *   seq_start, seq_len, entry : device int64 arrays [num]: listed entry k is entry
 *     entry[k] of the sequence occupying rows [seq_start[k], seq_start[k] + seq_len[k]);
 *     it reads rows seq_start[k] + m*entry[k] .. +m-1 (a) and the m rows before them (b,
 *     when entry[k] > 0), exactly as csa_compress does for that sequence.
 *   out : [num, c] out_dtype, row k = listed entry k.
 * The lists live in device memory and are not read on the host: each listed window is
 * checked on the device (0 <= seq_start, seq_start + seq_len <= total_rows,
 * 0 <= entry < seq_len / m); a failing entry is skipped, its output row is left
 * unwritten, and kvc_device_status() then reports KVC_ERR_INDEX. */
KVC_API kvc_status csa_compress_entries(const void* Ca, const void* Cb, const void* Za,
                                        const void* Zb, kvc_dtype in_dtype, const float* Ba,
                                        const float* Bb, int64_t total_rows, int64_t c,
                                        int32_t m, int32_t overlap, const int64_t* seq_start,
                                        const int64_t* seq_len, const int64_t* entry,
                                        int64_t num, void* out, kvc_dtype out_dtype,
                                        kvc_stream stream);

/* Entry lists for the HCA compressor: listed entry k pools rows
 * seq_start[k] + m*entry[k] .. +m-1 of the packed C, Z ([total_rows, c]); B : [m, c]. */
KVC_API kvc_status hca_compress_entries(const void* C, const void* Z, kvc_dtype in_dtype,
                                        const float* B, int64_t total_rows, int64_t c, int32_t m,
                                        const int64_t* seq_start, const int64_t* seq_len,
                                        const int64_t* entry, int64_t num, void* out,
                                        kvc_dtype out_dtype, kvc_stream stream);

/* Cache layout ([HCA] §4 (2): RoPE on the last r dimensions of each entry only, rotating
 * adjacent pairs of dimensions; the CSA/HCA comparison article's mixed-precision storage:
 * BF16 for the RoPE part, FP8 for the other KV values).  Instead of `out`, the entries are
 * written as
 *   out_nope : [rows, c - r] FP8 E4M3 bytes = entry[:c-r] * fp8_scale, rounded to nearest
 *              even, saturating at +-448 (16-byte aligned; unused when r == c)
 *   out_rope : [rows, r] bf16 = entry[c-r:] with pair j (dimensions 2j, 2j+1 of the slice)
 *              rotated by the angle pos * inv_freq[j], pos = pos_offset + pos_stride * i,
 *              i = the entry's index within its sequence (16-byte aligned; unused when r == 0)
 *   inv_freq : [r / 2] fp32 device array (the pages fix neither the frequencies nor the
 *              position a pooled entry takes: both are the caller's);  r % 8 == 0, 0 <= r <= c.
 * rows = batch * N_e for the dense calls, num for the entry-list calls.  The angle is
 * formed and reduced modulo 2 pi in fp64, its sine and cosine taken in fp32. */
KVC_API kvc_status csa_compress_cache(const void* Ca, const void* Cb, const void* Za,
                                      const void* Zb, kvc_dtype in_dtype, const float* Ba,
                                      const float* Bb, int64_t batch, int64_t n, int64_t c,
                                      int32_t m, int32_t overlap, int32_t r,
                                      const float* inv_freq, double pos_stride,
                                      double pos_offset, float fp8_scale, void* out_nope,
                                      void* out_rope, kvc_stream stream);
KVC_API kvc_status hca_compress_cache(const void* C, const void* Z, kvc_dtype in_dtype,
                                      const float* B, int64_t batch, int64_t n, int64_t c,
                                      int32_t m, int32_t r, const float* inv_freq,
                                      double pos_stride, double pos_offset, float fp8_scale,
                                      void* out_nope, void* out_rope, kvc_stream stream);
/* Entry lists written in the cache layout (decode-time cache insertion). */
KVC_API kvc_status csa_compress_entries_cache(
    const void* Ca, const void* Cb, const void* Za, const void* Zb, kvc_dtype in_dtype,
    const float* Ba, const float* Bb, int64_t total_rows, int64_t c, int32_t m, int32_t overlap,
    const int64_t* seq_start, const int64_t* seq_len, const int64_t* entry, int64_t num,
    int32_t r, const float* inv_freq, double pos_stride, double pos_offset, float fp8_scale,
    void* out_nope, void* out_rope, kvc_stream stream);
KVC_API kvc_status hca_compress_entries_cache(
    const void* C, const void* Z, kvc_dtype in_dtype, const float* B, int64_t total_rows,
    int64_t c, int32_t m, const int64_t* seq_start, const int64_t* seq_len,
    const int64_t* entry, int64_t num, int32_t r, const float* inv_freq, double pos_stride,
    double pos_offset, float fp8_scale, void* out_nope, void* out_rope, kvc_stream stream);

/* CSA compressor fed by hidden states ([SC] eq. attn-seqcomp-csa-proj followed by the
 * csa_compress pool): the four streams H W are formed on the tensor cores (bf16 in,
 * fp32 accumulate) and pooled on chip; they never reach device memory.
 *   H : [batch*n, d] bf16;  W_kva, W_kvb, W_za, W_zb : [d, c] bf16;  Ba, Bb : [m, c] fp32
 *   d % 64 == 0, c % 128 == 0;  out : [batch, N_e, c] out_dtype.
 *   The kernels implement the pages' CSA compressor only: m == 4 with overlap == 1.  Any
 *   other valid m or overlap = 0 returns KVC_ERR_UNSUPPORTED (before any launch); the
 *   streaming csa_compress covers those over precomputed streams. */
KVC_API kvc_status csa_compress_fused_proj(const void* H, const void* W_kva, const void* W_kvb,
                                   const void* W_za, const void* W_zb,
                                   const float* Ba, const float* Bb,
                                   int64_t batch, int64_t n, int64_t d, int64_t c,
                                   int32_t m, int32_t overlap,
                                   void* out, kvc_dtype out_dtype, kvc_stream stream);

/* HCA compressor fed by hidden states: C = H W_kv, Z = H W_z on the tensor cores, then
 * the hca_compress pool in the GEMM epilogue.  Shapes and rules as above; the kernels
 * implement m == 128 (the pages' m') only, any other valid m returns KVC_ERR_UNSUPPORTED. */
KVC_API kvc_status hca_compress_fused_proj(const void* H, const void* W_kv, const void* W_z,
                                   const float* B, int64_t batch, int64_t n, int64_t d,
                                   int64_t c, int32_t m,
                                   void* out, kvc_dtype out_dtype, kvc_stream stream);

/* The fused compressors in the scalar-logit form ([CSA] §3 symbol table: one score per
 * token and stream, z^a = H w^{Z_a} and z^b = H w^{Z_b} with w in R^d, an m-dimensional
 * bias, and one weight per window row shared by all channels; the streamed form is
 * csa_compress_scalar_logits).  C^a = H W_kva and C^b = H W_kvb are formed on the tensor
 * cores and the scores beside them; neither reaches device memory.
 *   H : [batch*n, d] bf16;  W_kva, W_kvb : [d, c] bf16;  w_za, w_zb : [d] bf16 (16-byte
 *   aligned);  ba, bb : [m] fp32;  out : [batch, N_e, c] out_dtype;  d % 64 == 0,
 *   c % 128 == 0; CSA m == 4 with overlap == 1, HCA m == 128, else KVC_ERR_UNSUPPORTED.
 *   Scores accumulate in fp32 from the bf16 products (exact in fp32). */
KVC_API kvc_status csa_compress_fused_proj_scalar(
    const void* H, const void* W_kva, const void* W_kvb, const void* w_za, const void* w_zb,
    const float* ba, const float* bb, int64_t batch, int64_t n, int64_t d, int64_t c, int32_t m,
    int32_t overlap, void* out, kvc_dtype out_dtype, kvc_stream stream);
/* HCA: C = H W_kv [d, c], z = H w_z [d], b : [m] fp32; entry i pools segment i. */
KVC_API kvc_status hca_compress_fused_proj_scalar(
    const void* H, const void* W_kv, const void* w_z, const float* b, int64_t batch, int64_t n,
    int64_t d, int64_t c, int32_t m, void* out, kvc_dtype out_dtype, kvc_stream stream);

/* The fused compressors with the entries written in the cache layout (the same layout as
 * csa_compress_cache above: [HCA] §4 (2) partial RoPE on the last r dimensions, the
 * comparison article's BF16 RoPE part and FP8 rest) straight from the GEMM epilogue ([SC]
 * flash-compressor section: RoPE and cache insertion are the fusions that sit next to the
 * compressor), so neither the streams nor the plain entries reach device memory.
 *   Arguments as csa_compress_fused_proj / hca_compress_fused_proj, with `out` and
 *   `out_dtype` replaced by r, inv_freq, pos_stride, pos_offset, fp8_scale, out_nope,
 *   out_rope as in csa_compress_cache (rows = batch * N_e; entry i of each sequence sits at
 *   position pos_offset + pos_stride * i).  The same m / overlap restrictions apply. */
KVC_API kvc_status csa_compress_fused_proj_cache(
    const void* H, const void* W_kva, const void* W_kvb, const void* W_za, const void* W_zb,
    const float* Ba, const float* Bb, int64_t batch, int64_t n, int64_t d, int64_t c, int32_t m,
    int32_t overlap, int32_t r, const float* inv_freq, double pos_stride, double pos_offset,
    float fp8_scale, void* out_nope, void* out_rope, kvc_stream stream);
KVC_API kvc_status hca_compress_fused_proj_cache(
    const void* H, const void* W_kv, const void* W_z, const float* B, int64_t batch, int64_t n,
    int64_t d, int64_t c, int32_t m, int32_t r, const float* inv_freq, double pos_stride,
    double pos_offset, float fp8_scale, void* out_nope, void* out_rope, kvc_stream stream);

/* ---------------------------------------------------------------- lightning indexer
 * [CSA] §4 (Lightning Indexer) and §5: CSA attends only to the compressed entries that
 * its indexer ranks highest.  Query t's score for compressed indexer key s is
 *     I[t, s] = sum_h w[t, h] * max(0, q[t, h] . K[s])
 * (one key per entry, shared by all indexer heads; 64 heads of width 128 on the page),
 * and the selected entries are those with the k largest scores (k = 1024 / 512).  The
 * keys are the compressed entries of an indexer compressor (csa_compress with c = 128).
 * Candidates.  Query t scores the n_visible[t] keys K[key_start[t] .. key_start[t] +
 *   n_visible[t] - 1] (its own sequence in a packed key array): a decode step passes all
 *   of its sequence's entries, a prefill query only the complete blocks before it.
 * Check on the device.  A query whose window leaves [0, key_rows) or whose n_visible
 *   exceeds max_visible is skipped (its rows untouched) and reported by
 *   kvc_device_status() as KVC_ERR_INDEX. */

/* Scores: scores[t * ld + s] = I[t, s] (fp32) for s < n_visible[t]; the rest of each
 * row is left untouched.
 *   q [T, H, D] bf16 with D == 128 and H a multiple of 16 in [16, 128];
 *   w [T, H] fp32 (4-byte aligned); K [key_rows, D] bf16;
 *   key_start, n_visible [T] int64 (8-byte aligned); scores [T, ld] fp32, ld >= max_visible;
 *   max_visible (host) an upper bound of every n_visible[t] (it sizes the launch).
 * q, K and scores are 16-byte aligned.  Dot products accumulate in fp32 on the tensor
 * cores (bf16 products are exact in fp32); ReLU and the head-weighted sum in fp32. */
KVC_API kvc_status lightning_indexer_scores(const void* q, const float* w, const void* K,
                                    const int64_t* key_start, const int64_t* n_visible,
                                    int64_t T, int32_t H, int32_t D, int64_t key_rows,
                                    int64_t max_visible, float* scores, int64_t ld,
                                    kvc_stream stream);

/* Top-k of each score row over its first n_visible[t] entries:
 *   out_idx[t * k + j] (int32), j < k: the entry indices in descending score order,
 *   equal scores by ascending index (-0.0 counts as 0.0); -1 for j >= n_visible[t].
 *   out_score[t * k + j] (fp32, may be NULL): the matching scores, -inf past the end.
 * 1 <= k <= 2048; max_visible <= kvc_topk_max_candidates(); scores [T, ld] fp32,
 * 16-byte aligned with ld a multiple of 4; n_visible as above.  The result is exact
 * for the given scores (no NaN among them).  The kernel is launched as a programmatic
 * dependent of the kernel ahead of it on the stream: it may start launching while that
 * kernel (lightning_indexer_scores in a decode step) finishes, and reads its inputs only
 * once that kernel has completed, so stream order holds as for any other call. */
KVC_API kvc_status indexer_topk(const float* scores, int64_t ld, const int64_t* n_visible,
                                int64_t T, int64_t max_visible, int32_t k, int32_t* out_idx,
                                float* out_score, kvc_stream stream);

/* The largest n_visible indexer_topk accepts (its candidates stay on chip). */
KVC_API int64_t kvc_topk_max_candidates(void);

/* Name of the kernel that the calling host thread's most recent successful call launched
 * (e.g. "csa_small_m_kernel/c512", "window_tma_kernel", "fused_pair_kernel/csa"); "" before
 * the first launch.  Static storage, never NULL.  The record is per host thread and is
 * left unchanged by calls that launch nothing (errors, empty problems).  It shows which
 * of the kernels behind one entry point the size-based dispatch picked. */
KVC_API const char* kvc_last_kernel(void);

/* Synchronises `stream`, then reports and clears the device-side error words that kernels
 * set: KVC_ERR_CUDA if the synchronisation or a read of the words failed; else
 * KVC_ERR_TIMEOUT if a bounded wait gave up (this takes precedence); else
 * KVC_ERR_WORKSPACE if a prepared-bias workspace did not match its call; else KVC_ERR_INDEX if
 * an entry list or an indexer window named rows outside its sequence or the streams; else
 * KVC_OK.  The words belong to the current device, not to a stream or a host thread: they
 * collect what every kernel of this library set since the last call, and one call clears
 * them for all callers. */
KVC_API kvc_status kvc_device_status(kvc_stream stream);

/* Sync check, off by default: with `on` nonzero, every call that launches work
 * synchronises its stream after the launch and returns what kvc_device_status() would
 * (KVC_ERR_TIMEOUT, KVC_ERR_WORKSPACE, KVC_ERR_INDEX, ...; the device error words are read
 * and cleared), so a kernel-side failure surfaces from the call that caused it.  A
 * debugging mode: it serialises the host with the stream.  Process-wide; a host-side
 * validation error is returned as before, without a synchronisation.  kvc_sync_check()
 * returns the current setting (0 or 1).  kvc_selftest_bounded_wait keeps reporting through
 * kvc_device_status() only. */
KVC_API void kvc_set_sync_check(int32_t on);
KVC_API int32_t kvc_sync_check(void);

/* Failure-detection self-test, no fault involved: launches one CTA whose first warp waits
 * on a shared-memory barrier that nothing completes, gives up after the kernels' wait limit
 * (2 s), raises the CTA's abort flag and the device error word; a second warp waiting on the
 * same barrier leaves as soon as it sees the flag.  out: device int32[2], written with
 * out[0] = 1 (the first wait gave up) and out[1] = 1 (the second left on the flag).
 * Afterwards kvc_device_status() reports KVC_ERR_TIMEOUT once and the context stays usable.
 * Errors: KVC_ERR_NULL, KVC_ERR_ALIGN, KVC_ERR_POINTER, KVC_ERR_CUDA (launch). */
KVC_API kvc_status kvc_selftest_bounded_wait(int32_t* out, kvc_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* KVC_H */
