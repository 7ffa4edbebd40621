// C ABI of the compressor: host-side validation, then one kernel launch per call.
// Every check here runs before anything is enqueued; see include/kvc.h for the contract.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "../../include/kvc.h"
#include "kvc_host.h"
#include "kvc_launch.h"

namespace {

using kvc::FusedProblem;
using kvc::StreamProblem;

constexpr int kMaxWindowRows = 320;  // longest window whose biases fit one CTA's shared memory

bool dtype_ok(kvc_dtype t) { return t == KVC_F32 || t == KVC_BF16; }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool mul_ok(int64_t a, int64_t b, int64_t* r) { return !__builtin_mul_overflow(a, b, r); }

// Device (or managed) memory of the current device.
kvc_status check_device_ptr(const void* p) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVC_ERR_CUDA;
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();  // clear the error this query leaves for unknown pointers
    return KVC_ERR_POINTER;
  }
  if (at.type == cudaMemoryTypeManaged) return KVC_OK;
  if (at.type != cudaMemoryTypeDevice || at.device != dev) return KVC_ERR_POINTER;
  return KVC_OK;
}

kvc_status check_ptrs(const void* const* ps, int n) {
  for (int i = 0; i < n; ++i) {
    kvc_status s = check_device_ptr(ps[i]);
    if (s != KVC_OK) return s;
  }
  return KVC_OK;
}

// Common shape checks of the streaming calls.  Sets *empty when nothing is to be done.
kvc_status check_stream_shape(int64_t batch, int64_t n, int64_t c, int32_t m, bool* empty,
                              int64_t* ne) {
  *empty = false;
  if (batch < 0 || n < 0 || c < 0 || m < 1) return KVC_ERR_SHAPE;
  *ne = n / m;
  int64_t t = 0;
  if (!mul_ok(batch, n, &t) || !mul_ok(t, c, &t) || !mul_ok(t, 4, &t)) return KVC_ERR_SHAPE;
  if (batch == 0 || *ne == 0 || c == 0) {
    *empty = true;
    return KVC_OK;
  }
  if (c % 8 != 0) return KVC_ERR_SHAPE;
  return KVC_OK;
}

// Checks and records the cache-layout arguments (after the problem's own checks).
template <typename Problem>
kvc_status set_cache(Problem* p, int32_t r, const float* inv_freq, double pos_stride,
                           double pos_offset, float fp8_scale, void* out_nope, void* out_rope) {
  if (r < 0 || r > p->c || r % 8 != 0) return KVC_ERR_SHAPE;
  if (!(fp8_scale == fp8_scale) || !(pos_stride == pos_stride) || !(pos_offset == pos_offset))
    return KVC_ERR_SHAPE;  // NaN arguments
  const bool has_nope = p->c - r > 0, has_rope = r > 0;
  if ((has_nope && !out_nope) || (has_rope && (!out_rope || !inv_freq))) return KVC_ERR_NULL;
  if ((has_nope && !aligned(out_nope, 16)) || (has_rope && !aligned(out_rope, 16)) ||
      (has_rope && !aligned(inv_freq, 4)))
    return KVC_ERR_ALIGN;
  const void* ps[3];
  int np = 0;
  if (has_nope) ps[np++] = out_nope;
  if (has_rope) {
    ps[np++] = out_rope;
    ps[np++] = inv_freq;
  }
  kvc_status s = check_ptrs(ps, np);
  if (s != KVC_OK) return s;
  p->cache = true;
  p->out_nope = out_nope;
  p->out_rope = out_rope;
  p->inv_freq = inv_freq;
  p->r = r;
  p->pos_stride = pos_stride;
  p->pos_offset = pos_offset;
  p->fp8_scale = fp8_scale;
  return KVC_OK;
}

}  // namespace

// Scratch of hca_compress_noalloc: the prepared-bias workspace lives here instead of in
// memory the caller allocates.  One array per device that loads the library, held until
// the process exits; every call on a device shares it.
constexpr int64_t kNoAllocScratchBytes = int64_t(1) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of g_noalloc_scratch on the current device.  In host code the array's
// name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress, once per device (with that device current), and kept.
kvc_status noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVC_ERR_CUDA;
  if (dev < 0 || dev >= 64) return KVC_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return KVC_ERR_CUDA;
    }
    addr[dev] = p;
  }
  *out = addr[dev];
  return KVC_OK;
}

// kvc_set_sync_check: process-wide, off by default.
std::atomic<int> g_sync_check{0};

// The status of a call that has launched its work: with the sync check on, the stream is
// synchronised and what the kernels reported is returned (as kvc_device_status would).
kvc_status finish(kvc_status launched, cudaStream_t st) {
  if (launched != KVC_OK || g_sync_check.load(std::memory_order_relaxed) == 0) return launched;
  return kvc::read_and_clear_device_error(st);
}

}  // namespace

extern "C" {

void kvc_set_sync_check(int32_t on) { g_sync_check.store(on != 0 ? 1 : 0); }

int32_t kvc_sync_check(void) { return g_sync_check.load(); }

int64_t kvc_num_entries(int64_t n, int32_t m) {
  if (n < 0 || m < 1) return -1;
  return n / m;
}

const char* kvc_status_string(kvc_status s) {
  switch (s) {
    case KVC_OK: return "KVC_OK";
    case KVC_ERR_NULL: return "KVC_ERR_NULL: a required pointer is NULL";
    case KVC_ERR_SHAPE: return "KVC_ERR_SHAPE: invalid size or shape";
    case KVC_ERR_DTYPE: return "KVC_ERR_DTYPE: unknown or unsupported dtype";
    case KVC_ERR_ALIGN: return "KVC_ERR_ALIGN: misaligned pointer";
    case KVC_ERR_UNSUPPORTED: return "KVC_ERR_UNSUPPORTED: valid but not implemented";
    case KVC_ERR_CUDA: return "KVC_ERR_CUDA: CUDA launch or query failed";
    case KVC_ERR_TIMEOUT: return "KVC_ERR_TIMEOUT: a bounded wait in a kernel gave up";
    case KVC_ERR_POINTER: return "KVC_ERR_POINTER: not device memory of the current device";
    case KVC_ERR_INDEX: return "KVC_ERR_INDEX: a listed entry was out of range and skipped";
    case KVC_ERR_WORKSPACE:
      return "KVC_ERR_WORKSPACE: the prepared-bias workspace was not made for this call";
    case KVC_ERR_TOO_LARGE:
      return "KVC_ERR_TOO_LARGE: the bias needs more than the 1 MiB fixed scratch of "
             "hca_compress_noalloc";
  }
  return "KVC_ERR_UNKNOWN";
}

kvc_status csa_compress(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                        kvc_dtype in_dtype, const float* Ba, const float* Bb, int64_t batch,
                        int64_t n, int64_t c, int32_t m, int32_t overlap, void* out,
                        kvc_dtype out_dtype, kvc_stream stream) {
  if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return KVC_ERR_DTYPE;
  if (overlap != 0 && overlap != 1) return KVC_ERR_SHAPE;
  bool empty = false;
  int64_t ne = 0;
  kvc_status s = check_stream_shape(batch, n, c, m, &empty, &ne);
  if (s != KVC_OK || empty) return s;
  if (!Ca || !Za || !Ba || !out) return KVC_ERR_NULL;
  if (overlap && (!Cb || !Zb || !Bb)) return KVC_ERR_NULL;
  if (!aligned(Ca, 16) || !aligned(Za, 16) || !aligned(out, 16) || !aligned(Ba, 4))
    return KVC_ERR_ALIGN;
  if (overlap && (!aligned(Cb, 16) || !aligned(Zb, 16) || !aligned(Bb, 4))) return KVC_ERR_ALIGN;
  const bool small = (m == 1 || m == 2 || m == 4);
  const int rows = overlap ? 2 * m : m;
  if (!small && rows > kMaxWindowRows) return KVC_ERR_UNSUPPORTED;
  {
    const void* ps[7] = {Ca, Za, Ba, out, Cb, Zb, Bb};
    s = check_ptrs(ps, overlap ? 7 : 4);
    if (s != KVC_OK) return s;
  }
  StreamProblem p{};
  p.C0 = Ca;
  p.Z0 = Za;
  p.B0 = Ba;
  p.C1 = overlap ? Cb : nullptr;
  p.Z1 = overlap ? Zb : nullptr;
  p.B1 = overlap ? Bb : nullptr;
  p.batch = batch;
  p.n = n;
  p.c = c;
  p.ne = ne;
  p.m = m;
  p.two_segments = overlap != 0;
  p.small_window_kernel = true;
  p.in_bf16 = in_dtype == KVC_BF16;
  p.out_bf16 = out_dtype == KVC_BF16;
  p.out = out;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_stream_pool(p, st), st);
}

kvc_status hca_compress(const void* C, const void* Z, kvc_dtype in_dtype, const float* B,
                        int64_t batch, int64_t n, int64_t c, int32_t m, void* out,
                        kvc_dtype out_dtype, kvc_stream stream) {
  if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return KVC_ERR_DTYPE;
  bool empty = false;
  int64_t ne = 0;
  kvc_status s = check_stream_shape(batch, n, c, m, &empty, &ne);
  if (s != KVC_OK || empty) return s;
  if (!C || !Z || !B || !out) return KVC_ERR_NULL;
  if (!aligned(C, 16) || !aligned(Z, 16) || !aligned(out, 16) || !aligned(B, 4))
    return KVC_ERR_ALIGN;
  if (m > kMaxWindowRows) return KVC_ERR_UNSUPPORTED;
  {
    const void* ps[4] = {C, Z, B, out};
    s = check_ptrs(ps, 4);
    if (s != KVC_OK) return s;
  }
  StreamProblem p{};
  p.C0 = C;
  p.Z0 = Z;
  p.B0 = B;
  p.batch = batch;
  p.n = n;
  p.c = c;
  p.ne = ne;
  p.m = m;
  p.two_segments = false;
  p.small_window_kernel = false;
  p.in_bf16 = in_dtype == KVC_BF16;
  p.out_bf16 = out_dtype == KVC_BF16;
  p.out = out;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_stream_pool(p, st), st);
}

int64_t hca_bias_workspace_bytes(int64_t c, int32_t m, kvc_dtype in_dtype) {
  if (c < 1 || m < 1 || !dtype_ok(in_dtype)) return -1;
  int64_t t = 0;
  if (!mul_ok(c, m + 1, &t) || !mul_ok(t, 8, &t)) return -1;
  return kvc::prep_layout(c, m, in_dtype == KVC_BF16).bytes;
}

kvc_status hca_prepare_bias(const float* B, int64_t c, int32_t m, kvc_dtype in_dtype,
                            void* workspace, int64_t workspace_bytes, kvc_stream stream) {
  if (!dtype_ok(in_dtype)) return KVC_ERR_DTYPE;
  if (c < 1 || m < 1 || c % 8 != 0) return KVC_ERR_SHAPE;
  if (m > kMaxWindowRows) return KVC_ERR_UNSUPPORTED;
  const int64_t need = hca_bias_workspace_bytes(c, m, in_dtype);
  if (need < 0 || workspace_bytes < need) return KVC_ERR_SHAPE;
  if (!B || !workspace) return KVC_ERR_NULL;
  if (!aligned(B, 4) || !aligned(workspace, 256)) return KVC_ERR_ALIGN;
  const void* ps[2] = {B, workspace};
  const kvc_status s = check_ptrs(ps, 2);
  if (s != KVC_OK) return s;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_prepare_bias(B, c, m, in_dtype == KVC_BF16, workspace, st), st);
}

kvc_status hca_compress_prepared(const void* C, const void* Z, kvc_dtype in_dtype,
                                 const void* workspace, int64_t workspace_bytes, int64_t batch,
                                 int64_t n, int64_t c, int32_t m, void* out, kvc_dtype out_dtype,
                                 kvc_stream stream) {
  if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return KVC_ERR_DTYPE;
  bool empty = false;
  int64_t ne = 0;
  kvc_status s = check_stream_shape(batch, n, c, m, &empty, &ne);
  if (s != KVC_OK || empty) return s;
  if (m > kMaxWindowRows) return KVC_ERR_UNSUPPORTED;
  const int64_t need = hca_bias_workspace_bytes(c, m, in_dtype);
  if (need < 0 || workspace_bytes < need) return KVC_ERR_SHAPE;
  if (!C || !Z || !workspace || !out) return KVC_ERR_NULL;
  if (!aligned(C, 16) || !aligned(Z, 16) || !aligned(out, 16) || !aligned(workspace, 256))
    return KVC_ERR_ALIGN;
  {
    const void* ps[4] = {C, Z, workspace, out};
    s = check_ptrs(ps, 4);
    if (s != KVC_OK) return s;
  }
  const kvc::PrepLayout l = kvc::prep_layout(c, m, in_dtype == KVC_BF16);
  StreamProblem p{};
  p.C0 = C;
  p.Z0 = Z;
  p.B0 = reinterpret_cast<const float*>(static_cast<const uint8_t*>(workspace) + l.raw_off);
  p.prep_ws = workspace;
  p.batch = batch;
  p.n = n;
  p.c = c;
  p.ne = ne;
  p.m = m;
  p.two_segments = false;
  p.small_window_kernel = false;
  p.in_bf16 = in_dtype == KVC_BF16;
  p.out_bf16 = out_dtype == KVC_BF16;
  p.out = out;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_stream_pool(p, st), st);
}

kvc_status hca_compress_noalloc(const void* C, const void* Z, kvc_dtype in_dtype, const float* B,
                                int64_t batch, int64_t n, int64_t c, int32_t m, void* out,
                                kvc_dtype out_dtype, kvc_stream stream) {
  if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return KVC_ERR_DTYPE;
  bool empty = false;
  int64_t ne = 0;
  kvc_status s = check_stream_shape(batch, n, c, m, &empty, &ne);
  if (s != KVC_OK || empty) return s;
  if (m > kMaxWindowRows) return KVC_ERR_UNSUPPORTED;
  const int64_t need = hca_bias_workspace_bytes(c, m, in_dtype);
  if (need < 0) return KVC_ERR_SHAPE;
  if (need > kNoAllocScratchBytes) return KVC_ERR_TOO_LARGE;
  if (!C || !Z || !B || !out) return KVC_ERR_NULL;
  if (!aligned(C, 16) || !aligned(Z, 16) || !aligned(out, 16) || !aligned(B, 4))
    return KVC_ERR_ALIGN;
  {
    const void* ps[4] = {C, Z, B, out};
    s = check_ptrs(ps, 4);
    if (s != KVC_OK) return s;
  }
  void* ws = nullptr;
  s = noalloc_scratch(&ws);
  if (s != KVC_OK) return s;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // every byte the compressor reads from the scratch is rewritten here first: nothing in
  // it needs to start at zero, and the previous call's contents are never read
  s = kvc::launch_prepare_bias(B, c, m, in_dtype == KVC_BF16, ws, st);
  if (s != KVC_OK) return s;
  const kvc::PrepLayout l = kvc::prep_layout(c, m, in_dtype == KVC_BF16);
  StreamProblem p{};
  p.C0 = C;
  p.Z0 = Z;
  p.B0 = reinterpret_cast<const float*>(static_cast<const uint8_t*>(ws) + l.raw_off);
  p.prep_ws = ws;
  p.batch = batch;
  p.n = n;
  p.c = c;
  p.ne = ne;
  p.m = m;
  p.two_segments = false;
  p.small_window_kernel = false;
  p.in_bf16 = in_dtype == KVC_BF16;
  p.out_bf16 = out_dtype == KVC_BF16;
  p.out = out;
  return finish(kvc::launch_stream_pool(p, st), st);
}

kvc_status csa_compress_scalar_logits(const void* Ca, const void* Cb, const void* za,
                                      const void* zb, kvc_dtype in_dtype, const float* ba,
                                      const float* bb, int64_t batch, int64_t n, int64_t c,
                                      int32_t m, int32_t overlap, void* out, kvc_dtype out_dtype,
                                      kvc_stream stream) {
  if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return KVC_ERR_DTYPE;
  if (overlap != 0 && overlap != 1) return KVC_ERR_SHAPE;
  bool empty = false;
  int64_t ne = 0;
  kvc_status s = check_stream_shape(batch, n, c, m, &empty, &ne);
  if (s != KVC_OK || empty) return s;
  if (!Ca || !za || !ba || !out) return KVC_ERR_NULL;
  if (overlap && (!Cb || !zb || !bb)) return KVC_ERR_NULL;
  const uintptr_t es = in_dtype == KVC_BF16 ? 2 : 4;
  if (!aligned(Ca, 16) || !aligned(out, 16) || !aligned(za, es) || !aligned(ba, 4))
    return KVC_ERR_ALIGN;
  if (overlap && (!aligned(Cb, 16) || !aligned(zb, es) || !aligned(bb, 4))) return KVC_ERR_ALIGN;
  if ((overlap ? 2 * m : m) > kMaxWindowRows) return KVC_ERR_UNSUPPORTED;
  {
    const void* ps[7] = {Ca, za, ba, out, Cb, zb, bb};
    s = check_ptrs(ps, overlap ? 7 : 4);
    if (s != KVC_OK) return s;
  }
  StreamProblem p{};
  p.C0 = Ca;
  p.Z0 = za;
  p.B0 = ba;
  p.C1 = overlap ? Cb : nullptr;
  p.Z1 = overlap ? zb : nullptr;
  p.B1 = overlap ? bb : nullptr;
  p.batch = batch;
  p.n = n;
  p.c = c;
  p.ne = ne;
  p.m = m;
  p.two_segments = overlap != 0;
  p.in_bf16 = in_dtype == KVC_BF16;
  p.out_bf16 = out_dtype == KVC_BF16;
  p.out = out;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_scalar_pool(p, st), st);
}

kvc_status hca_compress_scalar_logits(const void* C, const void* z, kvc_dtype in_dtype,
                                      const float* b, int64_t batch, int64_t n, int64_t c,
                                      int32_t m, void* out, kvc_dtype out_dtype,
                                      kvc_stream stream) {
  if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return KVC_ERR_DTYPE;
  bool empty = false;
  int64_t ne = 0;
  kvc_status s = check_stream_shape(batch, n, c, m, &empty, &ne);
  if (s != KVC_OK || empty) return s;
  if (!C || !z || !b || !out) return KVC_ERR_NULL;
  const uintptr_t es = in_dtype == KVC_BF16 ? 2 : 4;
  if (!aligned(C, 16) || !aligned(out, 16) || !aligned(z, es) || !aligned(b, 4))
    return KVC_ERR_ALIGN;
  if (m > kMaxWindowRows) return KVC_ERR_UNSUPPORTED;
  {
    const void* ps[4] = {C, z, b, out};
    s = check_ptrs(ps, 4);
    if (s != KVC_OK) return s;
  }
  StreamProblem p{};
  p.C0 = C;
  p.Z0 = z;
  p.B0 = b;
  p.batch = batch;
  p.n = n;
  p.c = c;
  p.ne = ne;
  p.m = m;
  p.two_segments = false;
  p.in_bf16 = in_dtype == KVC_BF16;
  p.out_bf16 = out_dtype == KVC_BF16;
  p.out = out;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_scalar_pool(p, st), st);
}

// Common checks of the entry-list calls; fills the list fields of p.
static kvc_status check_list(StreamProblem* p, int64_t total_rows, int64_t c, int32_t m,
                             const int64_t* seq_start, const int64_t* seq_len,
                             const int64_t* entry, int64_t num, bool* empty) {
  *empty = false;
  if (total_rows < 0 || c < 0 || m < 1 || num < 0) return KVC_ERR_SHAPE;
  int64_t t = 0;
  if (!mul_ok(total_rows, c, &t) || !mul_ok(t, 4, &t) || !mul_ok(num, c, &t)) return KVC_ERR_SHAPE;
  if (num == 0 || c == 0) {
    *empty = true;
    return KVC_OK;
  }
  if (c % 8 != 0) return KVC_ERR_SHAPE;
  if (!seq_start || !seq_len || !entry) return KVC_ERR_NULL;
  if (!aligned(seq_start, 8) || !aligned(seq_len, 8) || !aligned(entry, 8)) return KVC_ERR_ALIGN;
  p->listed = true;
  p->seq_start = seq_start;
  p->seq_len = seq_len;
  p->entry = entry;
  p->num = num;
  p->total_rows = total_rows;
  p->batch = 1;
  p->n = total_rows;
  p->c = c;
  p->ne = num;
  p->m = m;
  return KVC_OK;
}

kvc_status csa_compress_entries(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                                kvc_dtype in_dtype, const float* Ba, const float* Bb,
                                int64_t total_rows, int64_t c, int32_t m, int32_t overlap,
                                const int64_t* seq_start, const int64_t* seq_len,
                                const int64_t* entry, int64_t num, void* out,
                                kvc_dtype out_dtype, kvc_stream stream) {
  if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return KVC_ERR_DTYPE;
  if (overlap != 0 && overlap != 1) return KVC_ERR_SHAPE;
  StreamProblem p{};
  bool empty = false;
  kvc_status s = check_list(&p, total_rows, c, m, seq_start, seq_len, entry, num, &empty);
  if (s != KVC_OK || empty) return s;
  if (!Ca || !Za || !Ba || !out) return KVC_ERR_NULL;
  if (overlap && (!Cb || !Zb || !Bb)) return KVC_ERR_NULL;
  if (!aligned(Ca, 16) || !aligned(Za, 16) || !aligned(out, 16) || !aligned(Ba, 4))
    return KVC_ERR_ALIGN;
  if (overlap && (!aligned(Cb, 16) || !aligned(Zb, 16) || !aligned(Bb, 4))) return KVC_ERR_ALIGN;
  const bool small = (m == 1 || m == 2 || m == 4);
  if (!small && (overlap ? 2 * m : m) > kMaxWindowRows) return KVC_ERR_UNSUPPORTED;
  {
    const void* ps[10] = {Ca, Za, Ba, out, seq_start, seq_len, entry, Cb, Zb, Bb};
    s = check_ptrs(ps, overlap ? 10 : 7);
    if (s != KVC_OK) return s;
  }
  p.C0 = Ca;
  p.Z0 = Za;
  p.B0 = Ba;
  p.C1 = overlap ? Cb : nullptr;
  p.Z1 = overlap ? Zb : nullptr;
  p.B1 = overlap ? Bb : nullptr;
  p.two_segments = overlap != 0;
  p.small_window_kernel = true;
  p.in_bf16 = in_dtype == KVC_BF16;
  p.out_bf16 = out_dtype == KVC_BF16;
  p.out = out;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_stream_pool(p, st), st);
}

kvc_status hca_compress_entries(const void* C, const void* Z, kvc_dtype in_dtype, const float* B,
                                int64_t total_rows, int64_t c, int32_t m, const int64_t* seq_start,
                                const int64_t* seq_len, const int64_t* entry, int64_t num,
                                void* out, kvc_dtype out_dtype, kvc_stream stream) {
  if (!dtype_ok(in_dtype) || !dtype_ok(out_dtype)) return KVC_ERR_DTYPE;
  StreamProblem p{};
  bool empty = false;
  kvc_status s = check_list(&p, total_rows, c, m, seq_start, seq_len, entry, num, &empty);
  if (s != KVC_OK || empty) return s;
  if (!C || !Z || !B || !out) return KVC_ERR_NULL;
  if (!aligned(C, 16) || !aligned(Z, 16) || !aligned(out, 16) || !aligned(B, 4))
    return KVC_ERR_ALIGN;
  if (m > kMaxWindowRows) return KVC_ERR_UNSUPPORTED;
  {
    const void* ps[7] = {C, Z, B, out, seq_start, seq_len, entry};
    s = check_ptrs(ps, 7);
    if (s != KVC_OK) return s;
  }
  p.C0 = C;
  p.Z0 = Z;
  p.B0 = B;
  p.two_segments = false;
  p.small_window_kernel = false;
  p.in_bf16 = in_dtype == KVC_BF16;
  p.out_bf16 = out_dtype == KVC_BF16;
  p.out = out;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_stream_pool(p, st), st);
}

kvc_status csa_compress_cache(const void* Ca, const void* Cb, const void* Za, const void* Zb,
                              kvc_dtype in_dtype, const float* Ba, const float* Bb, int64_t batch,
                              int64_t n, int64_t c, int32_t m, int32_t overlap, int32_t r,
                              const float* inv_freq, double pos_stride, double pos_offset,
                              float fp8_scale, void* out_nope, void* out_rope, kvc_stream stream) {
  if (!dtype_ok(in_dtype)) return KVC_ERR_DTYPE;
  if (overlap != 0 && overlap != 1) return KVC_ERR_SHAPE;
  bool empty = false;
  int64_t ne = 0;
  kvc_status s = check_stream_shape(batch, n, c, m, &empty, &ne);
  if (s != KVC_OK || empty) return s;
  if (!Ca || !Za || !Ba) return KVC_ERR_NULL;
  if (overlap && (!Cb || !Zb || !Bb)) return KVC_ERR_NULL;
  if (!aligned(Ca, 16) || !aligned(Za, 16) || !aligned(Ba, 4)) return KVC_ERR_ALIGN;
  if (overlap && (!aligned(Cb, 16) || !aligned(Zb, 16) || !aligned(Bb, 4))) return KVC_ERR_ALIGN;
  const bool small = (m == 1 || m == 2 || m == 4);
  if (!small && (overlap ? 2 * m : m) > kMaxWindowRows) return KVC_ERR_UNSUPPORTED;
  StreamProblem p{};
  p.c = c;
  s = set_cache(&p, r, inv_freq, pos_stride, pos_offset, fp8_scale, out_nope, out_rope);
  if (s != KVC_OK) return s;
  {
    const void* ps[6] = {Ca, Za, Ba, Cb, Zb, Bb};
    s = check_ptrs(ps, overlap ? 6 : 3);
    if (s != KVC_OK) return s;
  }
  p.C0 = Ca;
  p.Z0 = Za;
  p.B0 = Ba;
  p.C1 = overlap ? Cb : nullptr;
  p.Z1 = overlap ? Zb : nullptr;
  p.B1 = overlap ? Bb : nullptr;
  p.batch = batch;
  p.n = n;
  p.ne = ne;
  p.m = m;
  p.two_segments = overlap != 0;
  p.small_window_kernel = true;
  p.in_bf16 = in_dtype == KVC_BF16;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_stream_pool(p, st), st);
}

kvc_status hca_compress_cache(const void* C, const void* Z, kvc_dtype in_dtype, const float* B,
                              int64_t batch, int64_t n, int64_t c, int32_t m, int32_t r,
                              const float* inv_freq, double pos_stride, double pos_offset,
                              float fp8_scale, void* out_nope, void* out_rope, kvc_stream stream) {
  if (!dtype_ok(in_dtype)) return KVC_ERR_DTYPE;
  bool empty = false;
  int64_t ne = 0;
  kvc_status s = check_stream_shape(batch, n, c, m, &empty, &ne);
  if (s != KVC_OK || empty) return s;
  if (!C || !Z || !B) return KVC_ERR_NULL;
  if (!aligned(C, 16) || !aligned(Z, 16) || !aligned(B, 4)) return KVC_ERR_ALIGN;
  if (m > kMaxWindowRows) return KVC_ERR_UNSUPPORTED;
  StreamProblem p{};
  p.c = c;
  s = set_cache(&p, r, inv_freq, pos_stride, pos_offset, fp8_scale, out_nope, out_rope);
  if (s != KVC_OK) return s;
  {
    const void* ps[3] = {C, Z, B};
    s = check_ptrs(ps, 3);
    if (s != KVC_OK) return s;
  }
  p.C0 = C;
  p.Z0 = Z;
  p.B0 = B;
  p.batch = batch;
  p.n = n;
  p.ne = ne;
  p.m = m;
  p.two_segments = false;
  p.small_window_kernel = false;
  p.in_bf16 = in_dtype == KVC_BF16;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_stream_pool(p, st), st);
}

kvc_status csa_compress_entries_cache(const void* Ca, const void* Cb, const void* Za,
                                      const void* Zb, kvc_dtype in_dtype, const float* Ba,
                                      const float* Bb, int64_t total_rows, int64_t c, int32_t m,
                                      int32_t overlap, const int64_t* seq_start,
                                      const int64_t* seq_len, const int64_t* entry, int64_t num,
                                      int32_t r, const float* inv_freq, double pos_stride,
                                      double pos_offset, float fp8_scale, void* out_nope,
                                      void* out_rope, kvc_stream stream) {
  if (!dtype_ok(in_dtype)) return KVC_ERR_DTYPE;
  if (overlap != 0 && overlap != 1) return KVC_ERR_SHAPE;
  StreamProblem p{};
  bool empty = false;
  kvc_status s = check_list(&p, total_rows, c, m, seq_start, seq_len, entry, num, &empty);
  if (s != KVC_OK || empty) return s;
  if (!Ca || !Za || !Ba) return KVC_ERR_NULL;
  if (overlap && (!Cb || !Zb || !Bb)) return KVC_ERR_NULL;
  if (!aligned(Ca, 16) || !aligned(Za, 16) || !aligned(Ba, 4)) return KVC_ERR_ALIGN;
  if (overlap && (!aligned(Cb, 16) || !aligned(Zb, 16) || !aligned(Bb, 4))) return KVC_ERR_ALIGN;
  const bool small = (m == 1 || m == 2 || m == 4);
  if (!small && (overlap ? 2 * m : m) > kMaxWindowRows) return KVC_ERR_UNSUPPORTED;
  s = set_cache(&p, r, inv_freq, pos_stride, pos_offset, fp8_scale, out_nope, out_rope);
  if (s != KVC_OK) return s;
  {
    const void* ps[9] = {Ca, Za, Ba, seq_start, seq_len, entry, Cb, Zb, Bb};
    s = check_ptrs(ps, overlap ? 9 : 6);
    if (s != KVC_OK) return s;
  }
  p.C0 = Ca;
  p.Z0 = Za;
  p.B0 = Ba;
  p.C1 = overlap ? Cb : nullptr;
  p.Z1 = overlap ? Zb : nullptr;
  p.B1 = overlap ? Bb : nullptr;
  p.two_segments = overlap != 0;
  p.small_window_kernel = true;
  p.in_bf16 = in_dtype == KVC_BF16;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_stream_pool(p, st), st);
}

kvc_status hca_compress_entries_cache(const void* C, const void* Z, kvc_dtype in_dtype,
                                      const float* B, int64_t total_rows, int64_t c, int32_t m,
                                      const int64_t* seq_start, const int64_t* seq_len,
                                      const int64_t* entry, int64_t num, int32_t r,
                                      const float* inv_freq, double pos_stride, double pos_offset,
                                      float fp8_scale, void* out_nope, void* out_rope,
                                      kvc_stream stream) {
  if (!dtype_ok(in_dtype)) return KVC_ERR_DTYPE;
  StreamProblem p{};
  bool empty = false;
  kvc_status s = check_list(&p, total_rows, c, m, seq_start, seq_len, entry, num, &empty);
  if (s != KVC_OK || empty) return s;
  if (!C || !Z || !B) return KVC_ERR_NULL;
  if (!aligned(C, 16) || !aligned(Z, 16) || !aligned(B, 4)) return KVC_ERR_ALIGN;
  if (m > kMaxWindowRows) return KVC_ERR_UNSUPPORTED;
  s = set_cache(&p, r, inv_freq, pos_stride, pos_offset, fp8_scale, out_nope, out_rope);
  if (s != KVC_OK) return s;
  {
    const void* ps[6] = {C, Z, B, seq_start, seq_len, entry};
    s = check_ptrs(ps, 6);
    if (s != KVC_OK) return s;
  }
  p.C0 = C;
  p.Z0 = Z;
  p.B0 = B;
  p.two_segments = false;
  p.small_window_kernel = false;
  p.in_bf16 = in_dtype == KVC_BF16;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_stream_pool(p, st), st);
}

// Device-memory check of the fused calls' inputs (and of `out` when non-NULL).
static kvc_status fused_ptrs(const void* H, const void* const* W, int nw, const float* B0,
                             const float* B1, const void* out) {
  const void* ps[3] = {H, B0, out};
  kvc_status s = check_ptrs(ps, out ? 3 : 2);
  if (s == KVC_OK) s = check_ptrs(W, nw);
  if (s == KVC_OK && B1) s = check_device_ptr(B1);
  return s;
}

// Common checks of the fused calls.  need_out: the plain output `out` is written (false
// for the cache layout, whose outputs set_cache checks; the inputs' device-memory check is
// then left to the caller, after the layout arguments have been checked).
static kvc_status fused_common(FusedProblem* p, bool csa, int32_t overlap, const void* H,
                               const void* const* W, int nw, const float* B0, const float* B1,
                               bool need_b1, int64_t batch, int64_t n, int64_t d, int64_t c,
                               int32_t m, void* out, kvc_dtype out_dtype, bool need_out,
                               bool* empty) {
  *empty = false;
  if (need_out && !dtype_ok(out_dtype)) return KVC_ERR_DTYPE;
  if (batch < 0 || n < 0 || d < 0 || c < 0 || m < 1) return KVC_ERR_SHAPE;
  int64_t t = 0;
  if (!mul_ok(batch, n, &t) || !mul_ok(t, d > c ? d : c, &t) || !mul_ok(t, 4, &t))
    return KVC_ERR_SHAPE;
  const int64_t ne = n / m;
  if (batch == 0 || ne == 0 || c == 0) {
    *empty = true;
    return KVC_OK;
  }
  if (d == 0 || d % 64 != 0 || c % 128 != 0) return KVC_ERR_SHAPE;
  // the tensor-core kernels implement the pages' two compressors only
  if (csa ? (m != 4 || overlap != 1) : m != 128) return KVC_ERR_UNSUPPORTED;
  if (!H || (need_out && !out) || !B0 || (need_b1 && !B1)) return KVC_ERR_NULL;
  for (int i = 0; i < nw; ++i)
    if (!W[i]) return KVC_ERR_NULL;
  if (!aligned(H, 16) || (need_out && !aligned(out, 16)) || !aligned(B0, 4)) return KVC_ERR_ALIGN;
  for (int i = 0; i < nw; ++i)
    if (!aligned(W[i], 16)) return KVC_ERR_ALIGN;
  if (need_b1 && !aligned(B1, 4)) return KVC_ERR_ALIGN;
  if (need_out) {
    const kvc_status s = fused_ptrs(H, W, nw, B0, need_b1 ? B1 : nullptr, out);
    if (s != KVC_OK) return s;
  }
  p->H = H;
  p->B0 = B0;
  p->B1 = need_b1 ? B1 : nullptr;
  p->batch = batch;
  p->n = n;
  p->d = d;
  p->c = c;
  p->ne = ne;
  p->m = m;
  p->out_bf16 = out_dtype == KVC_BF16;
  p->out = need_out ? out : nullptr;
  return KVC_OK;
}

kvc_status csa_compress_fused_proj(const void* H, const void* W_kva, const void* W_kvb,
                                   const void* W_za, const void* W_zb, const float* Ba,
                                   const float* Bb, int64_t batch, int64_t n, int64_t d,
                                   int64_t c, int32_t m, int32_t overlap, void* out,
                                   kvc_dtype out_dtype, kvc_stream stream) {
  if (overlap != 0 && overlap != 1) return KVC_ERR_SHAPE;
  FusedProblem p{};
  bool empty = false;
  kvc_status s;
  if (overlap) {
    const void* W[4] = {W_kva, W_kvb, W_za, W_zb};
    s = fused_common(&p, true, overlap, H, W, 4, Ba, Bb, true, batch, n, d, c, m, out, out_dtype,
                     true, &empty);
    for (int i = 0; i < 4; ++i) p.W[i] = W[i];
  } else {  // a-streams only
    const void* W[2] = {W_kva, W_za};
    s = fused_common(&p, true, overlap, H, W, 2, Ba, nullptr, false, batch, n, d, c, m, out,
                     out_dtype, true, &empty);
    p.W[0] = W_kva;
    p.W[1] = nullptr;
    p.W[2] = W_za;
    p.W[3] = nullptr;
  }
  if (s != KVC_OK || empty) return s;
  p.csa = true;
  p.overlap = overlap != 0;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_fused(p, st), st);
}

kvc_status hca_compress_fused_proj(const void* H, const void* W_kv, const void* W_z,
                                   const float* B, int64_t batch, int64_t n, int64_t d,
                                   int64_t c, int32_t m, void* out, kvc_dtype out_dtype,
                                   kvc_stream stream) {
  FusedProblem p{};
  bool empty = false;
  const void* W[2] = {W_kv, W_z};
  kvc_status s = fused_common(&p, false, 0, H, W, 2, B, nullptr, false, batch, n, d, c, m, out,
                              out_dtype, true, &empty);
  if (s != KVC_OK || empty) return s;
  p.W[0] = W_kv;
  p.W[1] = W_z;
  p.csa = false;
  p.overlap = false;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_fused(p, st), st);
}

kvc_status csa_compress_fused_proj_scalar(const void* H, const void* W_kva, const void* W_kvb,
                                          const void* w_za, const void* w_zb, const float* ba,
                                          const float* bb, int64_t batch, int64_t n, int64_t d,
                                          int64_t c, int32_t m, int32_t overlap, void* out,
                                          kvc_dtype out_dtype, kvc_stream stream) {
  if (overlap != 0 && overlap != 1) return KVC_ERR_SHAPE;
  FusedProblem p{};
  bool empty = false;
  const void* W[4] = {W_kva, W_kvb, w_za, w_zb};
  const kvc_status s = fused_common(&p, true, overlap, H, W, 4, ba, bb, true, batch, n, d, c, m,
                                    out, out_dtype, true, &empty);
  if (s != KVC_OK || empty) return s;
  p.W[0] = W_kva;
  p.W[1] = W_kvb;
  p.wz[0] = w_za;
  p.wz[1] = w_zb;
  p.scalar = true;
  p.csa = true;
  p.overlap = true;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_fused(p, st), st);
}

kvc_status hca_compress_fused_proj_scalar(const void* H, const void* W_kv, const void* w_z,
                                          const float* b, int64_t batch, int64_t n, int64_t d,
                                          int64_t c, int32_t m, void* out, kvc_dtype out_dtype,
                                          kvc_stream stream) {
  FusedProblem p{};
  bool empty = false;
  const void* W[2] = {W_kv, w_z};
  const kvc_status s = fused_common(&p, false, 0, H, W, 2, b, nullptr, false, batch, n, d, c, m,
                                    out, out_dtype, true, &empty);
  if (s != KVC_OK || empty) return s;
  p.W[0] = W_kv;
  p.wz[0] = w_z;
  p.wz[1] = w_z;
  p.scalar = true;
  p.csa = false;
  p.overlap = false;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_fused(p, st), st);
}

kvc_status csa_compress_fused_proj_cache(const void* H, const void* W_kva, const void* W_kvb,
                                         const void* W_za, const void* W_zb, const float* Ba,
                                         const float* Bb, int64_t batch, int64_t n, int64_t d,
                                         int64_t c, int32_t m, int32_t overlap, int32_t r,
                                         const float* inv_freq, double pos_stride,
                                         double pos_offset, float fp8_scale, void* out_nope,
                                         void* out_rope, kvc_stream stream) {
  if (overlap != 0 && overlap != 1) return KVC_ERR_SHAPE;
  FusedProblem p{};
  bool empty = false;
  const void* W[4] = {W_kva, W_kvb, W_za, W_zb};
  kvc_status s = fused_common(&p, true, overlap, H, W, 4, Ba, Bb, true, batch, n, d, c, m,
                              nullptr, KVC_BF16, false, &empty);
  if (s != KVC_OK || empty) return s;
  s = set_cache(&p, r, inv_freq, pos_stride, pos_offset, fp8_scale, out_nope, out_rope);
  if (s == KVC_OK) s = fused_ptrs(H, W, 4, Ba, Bb, nullptr);
  if (s != KVC_OK) return s;
  for (int i = 0; i < 4; ++i) p.W[i] = W[i];
  p.csa = true;
  p.overlap = true;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_fused(p, st), st);
}

kvc_status hca_compress_fused_proj_cache(const void* H, const void* W_kv, const void* W_z,
                                         const float* B, int64_t batch, int64_t n, int64_t d,
                                         int64_t c, int32_t m, int32_t r, const float* inv_freq,
                                         double pos_stride, double pos_offset, float fp8_scale,
                                         void* out_nope, void* out_rope, kvc_stream stream) {
  FusedProblem p{};
  bool empty = false;
  const void* W[2] = {W_kv, W_z};
  kvc_status s = fused_common(&p, false, 0, H, W, 2, B, nullptr, false, batch, n, d, c, m,
                              nullptr, KVC_BF16, false, &empty);
  if (s != KVC_OK || empty) return s;
  s = set_cache(&p, r, inv_freq, pos_stride, pos_offset, fp8_scale, out_nope, out_rope);
  if (s == KVC_OK) s = fused_ptrs(H, W, 2, B, nullptr, nullptr);
  if (s != KVC_OK) return s;
  p.W[0] = W_kv;
  p.W[1] = W_z;
  p.csa = false;
  p.overlap = false;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_fused(p, st), st);
}

kvc_status lightning_indexer_scores(const void* q, const float* w, const void* K,
                                    const int64_t* key_start, const int64_t* n_visible,
                                    int64_t T, int32_t H, int32_t D, int64_t key_rows,
                                    int64_t max_visible, float* scores, int64_t ld,
                                    kvc_stream stream) {
  if (T < 0 || key_rows < 0 || max_visible < 0 || ld < 0) return KVC_ERR_SHAPE;
  if (D != 128 || H < 16 || H > 128 || H % 16 != 0) return KVC_ERR_UNSUPPORTED;
  if (ld < max_visible) return KVC_ERR_SHAPE;
  int64_t tmp = 0;
  if (!mul_ok(T, ld, &tmp) || !mul_ok(tmp, 4, &tmp) || !mul_ok(T, H, &tmp) ||
      !mul_ok(key_rows, D * 2, &tmp))
    return KVC_ERR_SHAPE;
  if (T * H > (int64_t(1) << 31) - 1 || key_rows > (int64_t(1) << 31) - 1 - 256)
    return KVC_ERR_UNSUPPORTED;  // TMA row coordinates are 32-bit
  if (T == 0 || max_visible == 0) return KVC_OK;
  if (!q || !w || !K || !key_start || !n_visible || !scores) return KVC_ERR_NULL;
  if (!aligned(q, 16) || !aligned(K, 16) || !aligned(scores, 16) || !aligned(w, 4) ||
      !aligned(key_start, 8) || !aligned(n_visible, 8))
    return KVC_ERR_ALIGN;
  const void* ps[] = {q, w, K, key_start, n_visible, scores};
  kvc_status s = check_ptrs(ps, 6);
  if (s != KVC_OK) return s;
  kvc::IndexerProblem p{q, w, K, key_start, n_visible, T, key_rows, max_visible, ld, H, scores};
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_indexer_scores(p, st), st);
}

kvc_status indexer_topk(const float* scores, int64_t ld, const int64_t* n_visible, int64_t T,
                        int64_t max_visible, int32_t k, int32_t* out_idx, float* out_score,
                        kvc_stream stream) {
  if (T < 0 || max_visible < 0 || ld < 0 || k < 1) return KVC_ERR_SHAPE;
  if (k > 2048 || max_visible > kvc::topk_max_candidates()) return KVC_ERR_UNSUPPORTED;
  if (ld < max_visible || ld % 4 != 0) return KVC_ERR_SHAPE;
  int64_t tmp = 0;
  if (!mul_ok(T, ld, &tmp) || !mul_ok(tmp, 4, &tmp) || !mul_ok(T, k, &tmp) ||
      T > ((int64_t(1) << 31) - 1) / 8)
    return KVC_ERR_SHAPE;
  if (T == 0) return KVC_OK;
  if (!scores || !n_visible || !out_idx) return KVC_ERR_NULL;
  if (!aligned(scores, 16) || !aligned(n_visible, 8) || !aligned(out_idx, 4) ||
      (out_score && !aligned(out_score, 4)))
    return KVC_ERR_ALIGN;
  const void* ps[] = {scores, n_visible, out_idx};
  kvc_status s = check_ptrs(ps, 3);
  if (s == KVC_OK && out_score) s = check_device_ptr(out_score);
  if (s != KVC_OK) return s;
  kvc::TopkProblem p{scores, n_visible, T, max_visible, ld, k, out_idx, out_score};
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return finish(kvc::launch_indexer_topk(p, st), st);
}

int64_t kvc_topk_max_candidates(void) { return kvc::topk_max_candidates(); }

const char* kvc_last_kernel(void) { return kvc::last_kernel(); }

kvc_status kvc_device_status(kvc_stream stream) {
  return kvc::read_and_clear_device_error(reinterpret_cast<cudaStream_t>(stream));
}

kvc_status kvc_selftest_bounded_wait(int32_t* out, kvc_stream stream) {
  if (!out) return KVC_ERR_NULL;
  if (!aligned(out, 4)) return KVC_ERR_ALIGN;
  const kvc_status s = check_device_ptr(out);
  if (s != KVC_OK) return s;
  return kvc::launch_wait_selftest(out, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
