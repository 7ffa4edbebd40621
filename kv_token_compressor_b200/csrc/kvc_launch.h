// Internal launch interface between the C ABI (kvc_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/kvc.h"

namespace kvc {

// A validated streaming problem.  Segment 0 = (C0, Z0, B0): the a-range of CSA or the
// HCA segment; segment 1 = (C1, Z1, B1): the b-range of CSA with overlap.
struct StreamProblem {
  const void* C0;
  const void* Z0;
  const void* C1;
  const void* Z1;
  const float* B0;
  const float* B1;
  int64_t batch, n, c, ne;
  int m;
  bool two_segments;         // CSA with overlap
  bool small_window_kernel;  // allow the one-thread-per-entry kernel for m in {1,2,4}
  bool in_bf16, out_bf16;
  void* out;
  // Entry list (csa_compress_entries / hca_compress_entries): when `listed`, the kernel
  // compresses entry entry[k] of the sequence at rows [seq_start[k], +seq_len[k]) of the
  // packed streams (total_rows rows) into output row k, k < num; batch, n, ne unused.
  bool listed;
  const int64_t* seq_start;
  const int64_t* seq_len;
  const int64_t* entry;
  int64_t num, total_rows;
  // Cache layout (csa_compress_cache / hca_compress_cache): when `cache`, the entries go to
  // out_nope ([rows, c - r] E4M3) and out_rope ([rows, r] bf16) instead of `out`.
  bool cache;
  void* out_nope;
  void* out_rope;
  const float* inv_freq;
  int64_t r;
  double pos_stride, pos_offset;
  float fp8_scale;
  // Prepared bias (hca_compress_prepared): the workspace of hca_prepare_bias; B0 then points
  // at its raw copy of the bias.
  const void* prep_ws;
};

// Workspace of hca_prepare_bias, in this order: a 256-byte header, the raw bias [m, c] fp32
// (for the kernels that read plain rows), and for every channel slab of the TMA-fed window
// kernel (128 channels for bf16 streams, 64 for fp32) the block that kernel copies into its
// shared memory as it stands: the m rows scaled by log2 e in its consumers' float4 order
// (channels past c hold 0), the per-position maximum over the rows, and 4 floats whose
// first is 1 when every channel's spread max - min is within the fast-bound limit, else 0.
struct PrepHeader {
  uint32_t magic, version;
  int32_t m, in_bf16;
  int64_t c, slabs, slab_floats;  // slab block: (m + 1) * SC + 4 floats
  int64_t raw_off, prep_off;      // byte offsets from the workspace start
};
constexpr uint32_t kPrepMagic = 0x5052564Bu;
constexpr int64_t kPrepHeaderBytes = 256;
struct PrepLayout {
  int64_t sc, slabs, slab_floats, raw_off, prep_off, bytes;
};
inline PrepLayout prep_layout(int64_t c, int m, bool in_bf16) {
  PrepLayout l;
  l.sc = in_bf16 ? 128 : 64;
  l.slabs = (c + l.sc - 1) / l.sc;
  l.slab_floats = (static_cast<int64_t>(m) + 1) * l.sc + 4;
  l.raw_off = kPrepHeaderBytes;
  l.prep_off = l.raw_off + ((static_cast<int64_t>(m) * c * 4 + 255) / 256) * 256;
  l.bytes = l.prep_off + l.slabs * l.slab_floats * 4;
  return l;
}
// Fills a workspace (hca_prepare_bias); the caller has checked sizes and pointers.
kvc_status launch_prepare_bias(const float* B, int64_t c, int m, bool in_bf16, void* ws,
                               cudaStream_t st);

kvc_status launch_stream_pool(const StreamProblem& p, cudaStream_t st);
// Scalar-logit form: Z0 / Z1 point at [batch, n] logits, B0 / B1 at [m] biases.
kvc_status launch_scalar_pool(const StreamProblem& p, cudaStream_t st);
size_t window_kernel_smem_bytes(bool bf16_in, bool two_segments, int m);

// A validated fused problem: H [batch*n, d] bf16, W_s [d, c] bf16 (s = streams).
struct FusedProblem {
  const void* H;
  const void* W[4];  // CSA: kv_a, kv_b, z_a, z_b;  HCA: kv, z
  const float* B0;
  const float* B1;
  int64_t batch, n, d, c, ne;
  int m;
  bool csa;      // true: CSA (4 streams), false: HCA (2 streams)
  bool overlap;  // CSA only
  bool out_bf16;
  void* out;
  // Cache layout (the *_fused_proj_cache calls): when `cache`, the entries go to out_nope
  // ([rows, c - r] E4M3) and out_rope ([rows, r] bf16) instead of `out`.
  bool cache;
  void* out_nope;
  void* out_rope;
  const float* inv_freq;
  int64_t r;
  double pos_stride, pos_offset;
  float fp8_scale;
  // Scalar-logit form (the *_fused_proj_scalar calls): W[0] (and W[1] for CSA) are the value
  // projections, wz the score vectors [d] bf16, B0 / B1 the biases [m].
  bool scalar;
  const void* wz[2];
};

kvc_status launch_fused(const FusedProblem& p, cudaStream_t st);

// A validated lightning-indexer scoring problem (lightning_indexer_scores).
struct IndexerProblem {
  const void* q;  // [T, H, 128] bf16
  const float* w;  // [T, H]
  const void* K;  // [key_rows, 128] bf16
  const int64_t* key_start;
  const int64_t* n_visible;
  int64_t T, key_rows, max_visible, ld;
  int H;
  float* scores;  // [T, ld]
};
kvc_status launch_indexer_scores(const IndexerProblem& p, cudaStream_t st);

// A validated top-k problem (indexer_topk).
struct TopkProblem {
  const float* scores;  // [T, ld]
  const int64_t* n_visible;
  int64_t T, max_visible, ld;
  int k;
  int32_t* out_idx;   // [T, k]
  float* out_score;   // [T, k] or nullptr
};
kvc_status launch_indexer_topk(const TopkProblem& p, cudaStream_t st);
int64_t topk_max_candidates();
// Reads and clears the indexer kernels' error word (no synchronisation): bit 0 a bounded
// wait gave up, bit 1 a query's candidate window was out of range.
unsigned int read_and_clear_indexer_error(bool* failed);

// The TMA-fed single-segment window kernel (dense HCA-style problems with m >= 32);
// KVC_ERR_UNSUPPORTED when the problem or the device does not fit it (the caller then uses
// the register-staged kernels).
kvc_status launch_window_tma(const StreamProblem& p, cudaStream_t st);
// The TMA-fed CSA kernel (m = 4 with overlap, dense streams); KVC_ERR_UNSUPPORTED when the
// problem or the device does not fit it.
kvc_status launch_csa_tma(const StreamProblem& p, cudaStream_t st);
// The bounded-wait self-test kernel (kvc_selftest_bounded_wait).
kvc_status launch_wait_selftest(int32_t* out, cudaStream_t st);
// Reads and clears the TMA-fed kernels' error word (no synchronisation): bit 0 a bounded
// wait gave up.
unsigned int read_and_clear_window_error(bool* failed);

// Device error words: bounded waits that gave up (fused kernels) and listed entries out
// of range (streaming kernels).  Synchronises the stream first.
kvc_status read_and_clear_device_error(cudaStream_t st);
// Reads and clears the listed-entry error word (no synchronisation); true if it was set.
bool read_and_clear_index_error(bool* failed);

}  // namespace kvc
