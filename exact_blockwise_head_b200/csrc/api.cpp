// api.cpp -- the C ABI declared in include/attn.h: argument validation, path
// selection and the host copies of the tile rule.  Every check runs before
// anything is launched; nothing here allocates device memory or synchronises
// (except attn_device_status, which is documented to).
#include <cuda_runtime.h>

#include <cmath>
#include <cstddef>
#include <cstdint>
#include <mutex>

#include "attn.h"
#include "kernels.h"
#include "tiles.h"

namespace {

thread_local int g_last_cuda_error = 0;

constexpr uint64_t kDefaultTimeoutNs = 10ull * 1000 * 1000 * 1000;

int fail_cuda(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return ATTN_ERR_CUDA;
}

// Mask kinds that read `window`.
bool has_window(int mask_kind) {
  return mask_kind == ATTN_MASK_WINDOW || mask_kind == ATTN_MASK_CAUSAL_WINDOW;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Half-open byte ranges [a, a + na) and [b, b + nb) overlap?
bool overlap(const void* a, uint64_t na, const void* b, uint64_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Validation common to both paths; fills `out` with the normalised problem.
// check_overlap = false leaves the aliasing checks to a caller that knows the
// tensors' real extents (strided layouts).
int validate(const attn_params* p, ebh::FwdArgs* out, bool check_overlap = true) {
  if (p == nullptr) return ATTN_ERR_INVALID;
  if (p->dtype != ATTN_DTYPE_BF16 && p->dtype != ATTN_DTYPE_F32) return ATTN_ERR_INVALID;
  if (!p->q || !p->k || !p->v || !p->out) return ATTN_ERR_INVALID;
  if (p->B <= 0 || p->H <= 0 || p->L <= 0 || p->d <= 0) return ATTN_ERR_INVALID;
  if (static_cast<long long>(p->B) * p->H > 0x7fffffffLL) return ATTN_ERR_INVALID;
  if (!std::isfinite(p->scale) || !(p->scale > 0.f)) return ATTN_ERR_INVALID;
  if (p->mask_kind != ATTN_MASK_NONE && p->mask_kind != ATTN_MASK_CAUSAL &&
      p->mask_kind != ATTN_MASK_WINDOW && p->mask_kind != ATTN_MASK_CAUSAL_WINDOW)
    return ATTN_ERR_INVALID;
  if (has_window(p->mask_kind) && p->window < 0) return ATTN_ERR_INVALID;
  if (p->dtype == ATTN_DTYPE_BF16) {
    if (p->block_n != 0 && p->block_n != 64 && p->block_n != 128 && p->block_n != 256)
      return ATTN_ERR_INVALID;
  } else if (p->block_n != 0) {
    return ATTN_ERR_INVALID;
  }
  const uint64_t elem = p->dtype == ATTN_DTYPE_BF16 ? 2 : 4;
  const uint64_t rows = static_cast<uint64_t>(p->B) * p->H * p->L;
  const uint64_t tensor_bytes = rows * p->d * elem;
  const uint64_t lse_bytes = rows * 4;
  if (check_overlap && (overlap(p->out, tensor_bytes, p->q, tensor_bytes) ||
                        overlap(p->out, tensor_bytes, p->k, tensor_bytes) ||
                        overlap(p->out, tensor_bytes, p->v, tensor_bytes)))
    return ATTN_ERR_INVALID;
  if (check_overlap && p->lse && (overlap(p->lse, lse_bytes, p->q, tensor_bytes) ||
                 overlap(p->lse, lse_bytes, p->k, tensor_bytes) ||
                 overlap(p->lse, lse_bytes, p->v, tensor_bytes) ||
                 overlap(p->lse, lse_bytes, p->out, tensor_bytes)))
    return ATTN_ERR_INVALID;
  if (p->dtype == ATTN_DTYPE_BF16) {
    if (p->d != 64 && p->d != 128) return ATTN_ERR_UNSUPPORTED;
  } else if (p->d > 256) {
    return ATTN_ERR_UNSUPPORTED;
  }
  if (!aligned(p->q, 16) || !aligned(p->k, 16) || !aligned(p->v, 16) || !aligned(p->out, 16))
    return ATTN_ERR_MISALIGNED;
  if (p->lse && !aligned(p->lse, 4)) return ATTN_ERR_MISALIGNED;

  out->q = p->q;
  out->k = p->k;
  out->v = p->v;
  out->out = p->out;
  out->lse = p->lse;
  out->B = p->B;
  out->H = p->H;
  out->L = p->L;
  out->d = p->d;
  out->scale = p->scale;
  out->mask_kind = p->mask_kind;
  // a band at least L wide allows every pair: clamp so index sums stay small
  out->window = has_window(p->mask_kind) ? (p->window > p->L ? p->L : p->window) : 0;
  out->block_n = p->dtype == ATTN_DTYPE_BF16 ? (p->block_n == 0 ? 128 : p->block_n) : 0;
  out->timeout_ns = p->wait_timeout_ns ? p->wait_timeout_ns : kDefaultTimeoutNs;
  return ATTN_OK;
}

// The tensor-core path needs a compute-capability 10.0 device (sm_100a code).
int check_device_sm100() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e);
  static std::mutex mu;
  static int cc[64] = {0};
  std::lock_guard<std::mutex> g(mu);
  if (dev < 0 || dev >= 64) return fail_cuda(cudaErrorInvalidDevice);
  if (cc[dev] == 0) {
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) !=
        cudaSuccess)
      return fail_cuda(e);
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) !=
        cudaSuccess)
      return fail_cuda(e);
    cc[dev] = major * 10 + minor;
  }
  return cc[dev] == 100 ? ATTN_OK : ATTN_ERR_UNSUPPORTED;
}

}  // namespace

namespace ebh {
void set_last_cuda_error(cudaError_t e) { g_last_cuda_error = static_cast<int>(e); }

// Key runs the automatic choice takes: enough (query tile, run) units to
// cover the SMs once, at most ATTN_SPLITS_AUTO_MAX; with a causal mask at
// least two whenever the units fit in one wave (one unit per SM: the longest
// unit, the last rows, sets the time).  Balanced problems that already fill
// the SMs keep one run: they would only pay for the merge.
int auto_splits(long long units, bool causal, int nsm) {
  long long s = units > 0 ? nsm / units : 1;
  if (s < 1) s = 1;
  if (s > ATTN_SPLITS_AUTO_MAX) s = ATTN_SPLITS_AUTO_MAX;
  if (causal && units <= nsm && s < 2) s = 2;
  return static_cast<int>(s);
}

int current_sm_count(int* nsm) {
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess ||
      cudaDeviceGetAttribute(nsm, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return ATTN_ERR_CUDA;
  return ATTN_OK;
}

int splitkv_check(const attn_params* p, int num_splits, int* runs, int* run_blocks) {
  FwdArgs a;
  int st = validate(p, &a);
  if (st != ATTN_OK) return st;
  if (p->dtype != ATTN_DTYPE_BF16) return ATTN_ERR_UNSUPPORTED;
  if (num_splits < 0 || num_splits > kMaxSplits) return ATTN_ERR_INVALID;
  if (num_splits == ATTN_SPLITS_AUTO) {
    int nsm = 0;
    if ((st = current_sm_count(&nsm)) != ATTN_OK) return st;
    num_splits = attn_splitkv_auto_runs(a.B, a.H, a.L, a.mask_kind, nsm);
  }
  // whole key blocks per run; the last run may be shorter
  const int nkv = (a.L + a.block_n - 1) / a.block_n;
  *run_blocks = (nkv + num_splits - 1) / num_splits;
  *runs = (nkv + *run_blocks - 1) / *run_blocks;
  return ATTN_OK;
}
}  // namespace ebh

extern "C" {

int attn_fwd_ex(const attn_params* p, void* stream) {
  ebh::FwdArgs a;
  int st = validate(p, &a);
  if (st != ATTN_OK) return st;
  if ((st = check_device_sm100()) != ATTN_OK) return st;
  cudaError_t err = cudaSuccess;
  st = p->dtype == ATTN_DTYPE_BF16
           ? ebh::launch_fwd_bf16_sm100(a, static_cast<cudaStream_t>(stream), &err)
           : ebh::launch_fwd_f32(a, static_cast<cudaStream_t>(stream), &err);
  if (st == ATTN_ERR_CUDA) g_last_cuda_error = static_cast<int>(err);
  return st;
}

int attn_fwd_strided(const attn_params* p, const int64_t* strides, void* stream) {
  if (p == nullptr || strides == nullptr) return ATTN_ERR_INVALID;
  if (p->dtype != ATTN_DTYPE_BF16) return ATTN_ERR_UNSUPPORTED;
  ebh::FwdArgs a;
  int st = validate(p, &a, false);
  if (st != ATTN_OK) return st;
  // extent in bytes of each tensor: one past its last element
  uint64_t ext[4];
  for (int x = 0; x < 4; ++x) {
    const int64_t* s3 = strides + 3 * x;
    for (int y = 0; y < 3; ++y)
      if (s3[y] <= 0 || s3[y] % 8 != 0 || s3[y] > (int64_t(1) << 38)) return ATTN_ERR_INVALID;
    if (s3[0] < p->d) return ATTN_ERR_INVALID;
    ext[x] = (static_cast<uint64_t>(p->B - 1) * s3[2] + static_cast<uint64_t>(p->H - 1) * s3[1] +
              static_cast<uint64_t>(p->L - 1) * s3[0] + p->d) * 2;
    for (int y = 0; y < 3; ++y) a.stride[x][y] = s3[y];
  }
  const void* in[3] = {p->q, p->k, p->v};
  const uint64_t lse_bytes = static_cast<uint64_t>(p->B) * p->H * p->L * 4;
  for (int x = 0; x < 3; ++x) {
    if (overlap(p->out, ext[3], in[x], ext[x])) return ATTN_ERR_INVALID;
    if (p->lse && overlap(p->lse, lse_bytes, in[x], ext[x])) return ATTN_ERR_INVALID;
  }
  if (p->lse && overlap(p->lse, lse_bytes, p->out, ext[3])) return ATTN_ERR_INVALID;
  if ((st = check_device_sm100()) != ATTN_OK) return st;
  cudaError_t err = cudaSuccess;
  st = ebh::launch_fwd_bf16_sm100(a, static_cast<cudaStream_t>(stream), &err);
  if (st == ATTN_ERR_CUDA) g_last_cuda_error = static_cast<int>(err);
  return st;
}

int attn_fwd_rows(const attn_params* p, int kv_len, int q_offset, void* stream) {
  if (p == nullptr) return ATTN_ERR_INVALID;
  if (kv_len <= 0 || q_offset < 0 || p->L <= 0 ||
      static_cast<long long>(q_offset) + p->L > kv_len)
    return ATTN_ERR_INVALID;
  ebh::FwdArgs a;
  int st = validate(p, &a);
  if (st != ATTN_OK) return st;
  {  // k and v hold kv_len rows: check the outputs against their full extent
    const uint64_t elem = p->dtype == ATTN_DTYPE_BF16 ? 2 : 4;
    const uint64_t kv_bytes = static_cast<uint64_t>(p->B) * p->H * kv_len * p->d * elem;
    const uint64_t o_bytes = static_cast<uint64_t>(p->B) * p->H * p->L * p->d * elem;
    const uint64_t l_bytes = static_cast<uint64_t>(p->B) * p->H * p->L * 4;
    if (overlap(p->out, o_bytes, p->k, kv_bytes) || overlap(p->out, o_bytes, p->v, kv_bytes) ||
        (p->lse && (overlap(p->lse, l_bytes, p->k, kv_bytes) ||
                    overlap(p->lse, l_bytes, p->v, kv_bytes))))
      return ATTN_ERR_INVALID;
  }
  a.Lk = kv_len;
  a.q_shift = q_offset;
  // the band is measured in key positions: clamp it to the keys, not the rows
  a.window = has_window(p->mask_kind) ? (p->window > kv_len ? kv_len : p->window) : 0;
  if ((st = check_device_sm100()) != ATTN_OK) return st;
  cudaError_t err = cudaSuccess;
  st = p->dtype == ATTN_DTYPE_BF16
           ? ebh::launch_fwd_bf16_sm100(a, static_cast<cudaStream_t>(stream), &err)
           : ebh::launch_fwd_f32(a, static_cast<cudaStream_t>(stream), &err);
  if (st == ATTN_ERR_CUDA) g_last_cuda_error = static_cast<int>(err);
  return st;
}

int attn_seq_unshard(const void* gathered, void* out, int S, int B, int H, int Ls, int d,
                     int elem_bytes, void* stream) {
  if (!gathered || !out || S <= 0 || B <= 0 || H <= 0 || Ls <= 0 || d <= 0) return ATTN_ERR_INVALID;
  if (elem_bytes != 2 && elem_bytes != 4) return ATTN_ERR_INVALID;
  if (static_cast<long long>(B) * H > 0x7fffffffLL ||
      static_cast<long long>(S) * Ls > 0x7fffffffLL)
    return ATTN_ERR_INVALID;
  const uint64_t bytes = static_cast<uint64_t>(S) * B * H * Ls * d * elem_bytes;
  if (overlap(gathered, bytes, out, bytes)) return ATTN_ERR_INVALID;
  cudaError_t err = cudaSuccess;
  const int st = ebh::launch_unshard(gathered, out, S, B * H, Ls, d, elem_bytes,
                                     static_cast<cudaStream_t>(stream), &err);
  if (st == ATTN_ERR_CUDA) g_last_cuda_error = static_cast<int>(err);
  return st;
}

int attn_query_rows_for_keys(int L, int k_first, int k_last, int mask_kind, int window,
                             int* r_lo, int* r_hi) {
  if (!r_lo || !r_hi || L <= 0 || k_first < 0 || k_last < k_first || k_last >= L)
    return ATTN_ERR_INVALID;
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_CAUSAL_WINDOW) return ATTN_ERR_INVALID;
  if (has_window(mask_kind) && window < 0) return ATTN_ERR_INVALID;
  ebh::query_rows_for_keys(L, k_first, k_last, mask_kind, window, *r_lo, *r_hi);
  return ATTN_OK;
}

size_t attn_bwd_workspace_bytes(int B, int H, int L) {
  if (B <= 0 || H <= 0 || L <= 0) return 0;
  return static_cast<size_t>(B) * H * L * sizeof(float);
}

int attn_bwd(const attn_params* p, const void* dout, float* dq, float* dk, float* dv,
             void* workspace, size_t workspace_bytes, void* stream) {
  ebh::FwdArgs a;
  int st = validate(p, &a);
  if (st != ATTN_OK) return st;
  if (!p->lse || !dout || !dq || !dk || !dv || !workspace) return ATTN_ERR_INVALID;
  if (p->block_n != 0) return ATTN_ERR_INVALID;
  if (p->d > 128) return ATTN_ERR_UNSUPPORTED;
  const uint64_t rows = static_cast<uint64_t>(p->B) * p->H * p->L;
  const uint64_t elem = p->dtype == ATTN_DTYPE_BF16 ? 2 : 4;
  const uint64_t in_bytes = rows * p->d * elem;
  const uint64_t g_bytes = rows * p->d * 4;
  if (workspace_bytes < rows * 4) return ATTN_ERR_INVALID;
  if (!aligned(dout, 16) || !aligned(dq, 4) || !aligned(dk, 4) || !aligned(dv, 4) ||
      !aligned(workspace, 4))
    return ATTN_ERR_MISALIGNED;
  {  // the three gradients and the workspace must not overlap anything
    const void* outs[4] = {dq, dk, dv, workspace};
    const uint64_t out_sz[4] = {g_bytes, g_bytes, g_bytes, rows * 4};
    const void* ins[6] = {p->q, p->k, p->v, p->out, dout, p->lse};
    const uint64_t in_sz[6] = {in_bytes, in_bytes, in_bytes, in_bytes, in_bytes, rows * 4};
    for (int x = 0; x < 4; ++x) {
      for (int y = 0; y < 6; ++y)
        if (overlap(outs[x], out_sz[x], ins[y], in_sz[y])) return ATTN_ERR_INVALID;
      for (int y = x + 1; y < 4; ++y)
        if (overlap(outs[x], out_sz[x], outs[y], out_sz[y])) return ATTN_ERR_INVALID;
    }
  }
  if ((st = check_device_sm100()) != ATTN_OK) return st;
  ebh::BwdArgs b;
  b.q = p->q;
  b.k = p->k;
  b.v = p->v;
  b.out = p->out;
  b.dout = dout;
  b.lse = p->lse;
  b.D = static_cast<float*>(workspace);
  b.dq = dq;
  b.dk = dk;
  b.dv = dv;
  b.bf16 = p->dtype == ATTN_DTYPE_BF16;
  b.B = p->B;
  b.H = p->H;
  b.L = p->L;
  b.d = p->d;
  b.scale = p->scale;
  b.mask_kind = a.mask_kind;
  b.window = a.window;
  cudaError_t err = cudaSuccess;
  st = ebh::launch_bwd(b, static_cast<cudaStream_t>(stream), &err);
  if (st == ATTN_ERR_CUDA) g_last_cuda_error = static_cast<int>(err);
  return st;
}

size_t attn_mha_workspace_bytes(int B, int L, int E) {
  if (B <= 0 || L <= 0 || E <= 0) return 0;
  return ebh::mha_workspace_bytes(B, L, E);
}

int attn_mha_fwd(const attn_mha_params* p, void* workspace, size_t workspace_bytes,
                 void* stream) {
  if (p == nullptr || !p->x || !p->w_qkv || !p->w_out || !p->y || !workspace)
    return ATTN_ERR_INVALID;
  if (p->B <= 0 || p->L <= 0 || p->E <= 0 || p->H <= 0 || p->E % p->H != 0)
    return ATTN_ERR_INVALID;
  if (static_cast<long long>(p->B) * p->H > 0x7fffffffLL ||
      static_cast<long long>(p->B) * p->L > 0x7fffffffLL)
    return ATTN_ERR_INVALID;
  if (p->mask_kind < ATTN_MASK_NONE || p->mask_kind > ATTN_MASK_CAUSAL_WINDOW) return ATTN_ERR_INVALID;
  if (has_window(p->mask_kind) && p->window < 0) return ATTN_ERR_INVALID;
  const int d = p->E / p->H;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  const size_t need = ebh::mha_workspace_bytes(p->B, p->L, p->E);
  if (workspace_bytes < need) return ATTN_ERR_INVALID;
  if (!aligned(workspace, 256)) return ATTN_ERR_MISALIGNED;
  if (!aligned(p->x, 16) || !aligned(p->w_qkv, 16) || !aligned(p->w_out, 16) ||
      !aligned(p->y, 16) || (p->b_qkv && !aligned(p->b_qkv, 16)) ||
      (p->b_out && !aligned(p->b_out, 16)))
    return ATTN_ERR_MISALIGNED;
  {
    const uint64_t act = static_cast<uint64_t>(p->B) * p->L * p->E * 2;
    const uint64_t wq = static_cast<uint64_t>(3) * p->E * p->E * 2;
    const uint64_t wo = static_cast<uint64_t>(p->E) * p->E * 2;
    if (overlap(workspace, need, p->x, act) || overlap(workspace, need, p->y, act) ||
        overlap(workspace, need, p->w_qkv, wq) || overlap(workspace, need, p->w_out, wo) ||
        overlap(p->y, act, p->x, act) || overlap(p->y, act, p->w_qkv, wq) ||
        overlap(p->y, act, p->w_out, wo))
      return ATTN_ERR_INVALID;
  }
  int st = check_device_sm100();
  if (st != ATTN_OK) return st;
  ebh::MhaArgs a;
  a.x = p->x;
  a.w_qkv = p->w_qkv;
  a.b_qkv = p->b_qkv;
  a.w_out = p->w_out;
  a.b_out = p->b_out;
  a.y = p->y;
  a.B = p->B;
  a.L = p->L;
  a.E = p->E;
  a.H = p->H;
  a.scale = 1.0f / std::sqrt(static_cast<float>(d));
  a.mask_kind = p->mask_kind;
  a.window = has_window(p->mask_kind) ? (p->window > p->L ? p->L : p->window) : 0;
  a.timeout_ns = kDefaultTimeoutNs;
  cudaError_t err = cudaSuccess;
  int proj = 0;
  st = ebh::launch_mha(a, workspace, static_cast<cudaStream_t>(stream), &err, &proj);
  if (st == ATTN_ERR_CUDA) g_last_cuda_error = static_cast<int>(err);
  return st;
}

int attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H,
             int L, int d, float scale, int mask_kind, int window, void* stream) {
  attn_params p = {};
  p.dtype = ATTN_DTYPE_BF16;
  p.q = q;
  p.k = k;
  p.v = v;
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.L = L;
  p.d = d;
  p.scale = scale;
  p.mask_kind = mask_kind;
  p.window = window;
  return attn_fwd_ex(&p, stream);
}

int attn_fwd_f32(const float* q, const float* k, const float* v, float* out, float* lse, int B,
                 int H, int L, int d, float scale, int mask_kind, int window, void* stream) {
  attn_params p = {};
  p.dtype = ATTN_DTYPE_F32;
  p.q = q;
  p.k = k;
  p.v = v;
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.L = L;
  p.d = d;
  p.scale = scale;
  p.mask_kind = mask_kind;
  p.window = window;
  return attn_fwd_ex(&p, stream);
}

const char* attn_strerror(int status) {
  switch (status) {
    case ATTN_OK: return "success";
    case ATTN_ERR_INVALID: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported head dimension, size or device";
    case ATTN_ERR_MISALIGNED: return "misaligned pointer (q/k/v/out need 16 bytes, lse 4)";
    case ATTN_ERR_CUDA: return "CUDA runtime error (see attn_last_cuda_error)";
    case ATTN_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
    case ATTN_ERR_SCRATCH_LIMIT:
      return "problem needs more scratch than the fixed no-allocation scratch "
             "(ATTN_NOALLOC_SCRATCH_BYTES) holds";
    default: return "unknown status";
  }
}

int attn_last_cuda_error(void) { return g_last_cuda_error; }

int attn_device_status(int device, int reset) {
  cudaError_t err = cudaSuccess;
  int st = ebh::read_device_status(device, reset, &err);
  if (st == ATTN_ERR_CUDA) g_last_cuda_error = static_cast<int>(err);
  return st;
}

int attn_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns == 0) return ATTN_ERR_INVALID;
  int st = check_device_sm100();
  if (st != ATTN_OK) return st;
  cudaError_t err = cudaSuccess;
  st = ebh::launch_selftest_wait_timeout(limit_ns, static_cast<cudaStream_t>(stream), &err);
  if (st == ATTN_ERR_CUDA) g_last_cuda_error = static_cast<int>(err);
  return st;
}

int attn_kv_tile_range(int L, int q_first, int q_last, int mask_kind, int window, int block_n,
                       int* lo, int* hi) {
  if (!lo || !hi || L <= 0 || block_n <= 0 || q_first < 0 || q_last < q_first || q_last >= L)
    return ATTN_ERR_INVALID;
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_CAUSAL_WINDOW) return ATTN_ERR_INVALID;
  if (has_window(mask_kind) && window < 0) return ATTN_ERR_INVALID;
  ebh::kv_tile_range(L, q_first, q_last, mask_kind, window, block_n, *lo, *hi);
  return ATTN_OK;
}

int attn_kv_tile_class(int L, int q_first, int q_last, int j, int mask_kind, int window,
                       int block_n) {
  if (L <= 0 || block_n <= 0 || q_first < 0 || q_last < q_first || q_last >= L)
    return -ATTN_ERR_INVALID;
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_CAUSAL_WINDOW) return -ATTN_ERR_INVALID;
  if (has_window(mask_kind) && window < 0) return -ATTN_ERR_INVALID;
  return ebh::kv_tile_class(L, q_first, q_last, j, mask_kind, window, block_n);
}

int attn_splitkv_auto_runs(int B, int H, int L, int mask_kind, int num_sms) {
  if (B < 1 || H < 1 || L < 1 || num_sms < 1 || mask_kind < ATTN_MASK_NONE ||
      mask_kind > ATTN_MASK_CAUSAL_WINDOW)
    return 0;
  const long long units = static_cast<long long>(B) * H * ((static_cast<long long>(L) + 255) / 256);
  return ebh::auto_splits(units, mask_kind == ATTN_MASK_CAUSAL, num_sms);
}

size_t attn_splitkv_workspace_bytes(int B, int H, int L, int d, int num_splits) {
  if (B <= 0 || H <= 0 || L <= 0 || d <= 0) return 0;
  if (num_splits == ATTN_SPLITS_AUTO) {
    // the current device's choice for a causal mask, which is never below
    // that for any other mask; without a device, the most it could choose
    int nsm = 0;
    num_splits = ebh::current_sm_count(&nsm) == ATTN_OK
                     ? attn_splitkv_auto_runs(B, H, L, ATTN_MASK_CAUSAL, nsm)
                     : ATTN_SPLITS_AUTO_MAX;
  }
  if (num_splits < 1) return 0;
  const size_t rows = static_cast<size_t>(num_splits) * B * H * L;
  const size_t o_bytes = (rows * d * sizeof(float) + 255) / 256 * 256;
  return o_bytes + rows * sizeof(float);
}

int attn_fwd_splitkv(const attn_params* p, int num_splits, void* workspace,
                     size_t workspace_bytes, void* stream) {
  int splits = 0, split_blocks = 0;
  int st = ebh::splitkv_check(p, num_splits, &splits, &split_blocks);
  if (st != ATTN_OK) return st;
  if (splits == 1) return attn_fwd_ex(p, stream);
  ebh::FwdArgs a;
  if ((st = validate(p, &a)) != ATTN_OK) return st;
  const size_t need = attn_splitkv_workspace_bytes(a.B, a.H, a.L, a.d, splits);
  if (workspace == nullptr || workspace_bytes < need) return ATTN_ERR_INVALID;
  if (!aligned(workspace, 256)) return ATTN_ERR_MISALIGNED;
  const size_t rows = static_cast<size_t>(splits) * a.B * a.H * a.L;
  const size_t o_bytes = (rows * a.d * sizeof(float) + 255) / 256 * 256;
  float* o_part = static_cast<float*>(workspace);
  float* lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + o_bytes);
  {  // the workspace must not alias the problem's tensors
    const uint64_t tb = static_cast<uint64_t>(a.B) * a.H * a.L * a.d * 2;
    const uint64_t lb = static_cast<uint64_t>(a.B) * a.H * a.L * 4;
    if (overlap(workspace, need, p->q, tb) || overlap(workspace, need, p->k, tb) ||
        overlap(workspace, need, p->v, tb) || overlap(workspace, need, p->out, tb) ||
        (p->lse && overlap(workspace, need, p->lse, lb)))
      return ATTN_ERR_INVALID;
  }
  if ((st = check_device_sm100()) != ATTN_OK) return st;
  a.num_splits = splits;
  a.split_keys = split_blocks * a.block_n;
  a.o_part = o_part;
  a.lse_part = lse_part;
  cudaError_t err = cudaSuccess;
  st = ebh::launch_fwd_bf16_sm100(a, static_cast<cudaStream_t>(stream), &err);
  if (st != ATTN_OK) {
    if (st == ATTN_ERR_CUDA) g_last_cuda_error = static_cast<int>(err);
    return st;
  }
  ebh::MergeArgs m = {};
  m.o_part = o_part;
  m.lse_part = lse_part;
  m.num_splits = splits;
  for (int s = 0; s <= splits; ++s) {
    const long long b = static_cast<long long>(s) * a.split_keys;
    m.bounds[s] = static_cast<int>(b < a.L ? b : a.L);
  }
  m.out = a.out;
  m.lse = a.lse;
  m.out_f32 = false;
  m.BH = a.B * a.H;
  m.L = a.L;
  m.d = a.d;
  m.mask_kind = a.mask_kind;
  m.window = a.window;
  m.kv_len = a.L;
  m.q_offset = 0;
  m.dependent = true;  // the partial kernel just before it on the stream
  st = ebh::launch_merge(m, static_cast<cudaStream_t>(stream), &err);
  if (st == ATTN_ERR_CUDA) g_last_cuda_error = static_cast<int>(err);
  return st;
}

int attn_merge_rows(const float* o_parts, const float* lse_parts, int num_splits,
                    const int* split_bounds, int mask_kind, int window, void* out, float* lse,
                    int out_dtype, int B, int H, int L, int d, int kv_len, int q_offset,
                    void* stream) {
  if (!o_parts || !lse_parts || !split_bounds || !out) return ATTN_ERR_INVALID;
  if (num_splits < 1 || num_splits > ebh::kMaxSplits) return ATTN_ERR_INVALID;
  if (B <= 0 || H <= 0 || L <= 0 || kv_len <= 0) return ATTN_ERR_INVALID;
  if (static_cast<long long>(B) * H > 0x7fffffffLL) return ATTN_ERR_INVALID;
  if (q_offset < 0 || static_cast<long long>(q_offset) + L > kv_len) return ATTN_ERR_INVALID;
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_CAUSAL_WINDOW) return ATTN_ERR_INVALID;
  if (has_window(mask_kind) && window < 0) return ATTN_ERR_INVALID;
  if (out_dtype != ATTN_DTYPE_BF16 && out_dtype != ATTN_DTYPE_F32) return ATTN_ERR_INVALID;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (split_bounds[0] != 0) return ATTN_ERR_INVALID;
  for (int s = 0; s < num_splits; ++s)
    if (split_bounds[s + 1] < split_bounds[s]) return ATTN_ERR_INVALID;
  if (split_bounds[num_splits] != kv_len) return ATTN_ERR_INVALID;
  if (!aligned(o_parts, 16) || !aligned(lse_parts, 4) || !aligned(out, 16) ||
      (lse && !aligned(lse, 4)))
    return ATTN_ERR_MISALIGNED;
  int st = check_device_sm100();
  if (st != ATTN_OK) return st;
  ebh::MergeArgs m = {};
  m.o_part = o_parts;
  m.lse_part = lse_parts;
  m.num_splits = num_splits;
  for (int s = 0; s <= num_splits; ++s) m.bounds[s] = split_bounds[s];
  m.out = out;
  m.lse = lse;
  m.out_f32 = out_dtype == ATTN_DTYPE_F32;
  m.BH = B * H;
  m.L = L;
  m.d = d;
  m.mask_kind = mask_kind;
  m.window = has_window(mask_kind) ? (window > kv_len ? kv_len : window) : 0;
  m.kv_len = kv_len;
  m.q_offset = q_offset;
  cudaError_t err = cudaSuccess;
  st = ebh::launch_merge(m, static_cast<cudaStream_t>(stream), &err);
  if (st == ATTN_ERR_CUDA) g_last_cuda_error = static_cast<int>(err);
  return st;
}

int attn_merge(const float* o_parts, const float* lse_parts, int num_splits,
               const int* split_bounds, int mask_kind, int window, void* out, float* lse,
               int out_dtype, int B, int H, int L, int d, void* stream) {
  return attn_merge_rows(o_parts, lse_parts, num_splits, split_bounds, mask_kind, window, out, lse,
                         out_dtype, B, H, L, d, L, 0, stream);
}

int attn_fwd_partial(const attn_params* p, int kv_len, int q_shift, float* o_part,
                     float* lse_part, void* stream) {
  if (p == nullptr || o_part == nullptr || lse_part == nullptr) return ATTN_ERR_INVALID;
  if (p->dtype != ATTN_DTYPE_BF16) return ATTN_ERR_UNSUPPORTED;
  if (kv_len <= 0) return ATTN_ERR_INVALID;
  // every key position a row could reach stays inside int: |shift| + L + kv_len
  const long long reach = (q_shift < 0 ? -static_cast<long long>(q_shift) : q_shift) +
                          static_cast<long long>(p->L) + kv_len;
  if (reach > 0x3fffffffLL) return ATTN_ERR_INVALID;
  // p->out and p->lse are not used: the results go to o_part and lse_part
  attn_params pc = *p;
  pc.out = o_part;
  pc.lse = nullptr;
  ebh::FwdArgs a;
  int st = validate(&pc, &a);
  if (st != ATTN_OK) return st;
  {  // k and v hold kv_len rows; the partials must not overlap anything
    const uint64_t rows = static_cast<uint64_t>(p->B) * p->H * p->L;
    const uint64_t kv_bytes = static_cast<uint64_t>(p->B) * p->H * kv_len * p->d * 2;
    const uint64_t o_bytes = rows * p->d * 4, l_bytes = rows * 4;
    const uint64_t q_bytes = rows * p->d * 2;
    if (!aligned(o_part, 16) || !aligned(lse_part, 4)) return ATTN_ERR_MISALIGNED;
    const void* ins[3] = {p->q, p->k, p->v};
    const uint64_t in_sz[3] = {q_bytes, kv_bytes, kv_bytes};
    for (int x = 0; x < 3; ++x)
      if (overlap(o_part, o_bytes, ins[x], in_sz[x]) || overlap(lse_part, l_bytes, ins[x], in_sz[x]))
        return ATTN_ERR_INVALID;
    if (overlap(o_part, o_bytes, lse_part, l_bytes)) return ATTN_ERR_INVALID;
  }
  a.Lk = kv_len;
  a.q_shift = q_shift;
  // a band wider than any distance between a row and a key allows every pair
  a.window = has_window(p->mask_kind) ? static_cast<int>(p->window > reach ? reach : p->window)
                                      : 0;
  const int nkv = (kv_len + a.block_n - 1) / a.block_n;
  a.num_splits = 1;  // one run over all of the given keys, written as a partial
  a.split_keys = nkv * a.block_n;
  a.o_part = o_part;
  a.lse_part = lse_part;
  if ((st = check_device_sm100()) != ATTN_OK) return st;
  cudaError_t err = cudaSuccess;
  st = ebh::launch_fwd_bf16_sm100(a, static_cast<cudaStream_t>(stream), &err);
  if (st == ATTN_ERR_CUDA) g_last_cuda_error = static_cast<int>(err);
  return st;
}

int attn_kv_full_range(int L, int q_first, int q_last, int mask_kind, int window, int block_n,
                       int* lo, int* hi) {
  if (!lo || !hi || L <= 0 || block_n <= 0 || q_first < 0 || q_last < q_first || q_last >= L)
    return ATTN_ERR_INVALID;
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_CAUSAL_WINDOW) return ATTN_ERR_INVALID;
  if (has_window(mask_kind) && window < 0) return ATTN_ERR_INVALID;
  ebh::kv_full_range(L, q_first, q_last, mask_kind, window, block_n, *lo, *hi);
  return ATTN_OK;
}

int attn_abi_version(void) { return ATTN_ABI_VERSION; }

}  // extern "C"
