// mha.cu -- the multi-head attention layer around the attention kernel.
//
// "Transformer multi-head attention, 8-head parallel computation" (lshu.cn),
// sections 2.1 and 2.2, builds the layer as
//   qkv = x W_qkv^T + b_qkv            (one Linear(E, 3E))
//   q, k, v = the three E-wide thirds of qkv, each viewed [B, L, H, d] and
//             transposed to [B, H, L, d]  (d = E / H)
//   context = softmax(q k^T / sqrt(d) + mask) v, transposed back to [B, L, E]
//   y = context W_out^T + b_out        (one Linear(E, E))
// The two projections are plain GEMMs and run in cuBLASLt (bf16 operands,
// fp32 accumulation, the bias added in its epilogue).  The attention kernel
// reads q, k and v straight out of the projection's [B, L, 3, H, d] output
// through strided tensor maps and writes the context in [B, L, H, d], so the
// head split and merge cost no pass of their own.
#include <cublasLt.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "attn.h"
#include "kernels.h"

namespace ebh {
namespace {

constexpr size_t kLtWorkspace = size_t(32) << 20;

cublasLtHandle_t lt_handle(int device, cublasStatus_t* st) {
  static std::mutex mu;
  static cublasLtHandle_t handles[64] = {};
  std::lock_guard<std::mutex> g(mu);
  *st = CUBLAS_STATUS_SUCCESS;
  if (device < 0 || device >= 64) {
    *st = CUBLAS_STATUS_INVALID_VALUE;
    return nullptr;
  }
  if (handles[device] == nullptr) *st = cublasLtCreate(&handles[device]);
  return handles[device];
}

// Row-major Y[M, N] = X[M, K] W[N, K]^T + bias[N] (bias may be null), all bf16,
// fp32 accumulation.  In column-major terms: Y^T (N x M) = W (N x K) X^T.
bool linear_bf16(cublasLtHandle_t h, const void* X, const void* W, const void* bias, void* Y,
                 int M, int N, int K, void* lt_ws, cudaStream_t stream) {
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  bool ok = false;
  do {
    if (cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS)
      break;
    const cublasOperation_t ta = CUBLAS_OP_T, tb = CUBLAS_OP_N;
    cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &ta, sizeof(ta));
    cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &tb, sizeof(tb));
    if (bias != nullptr) {
      const cublasLtEpilogue_t epi = CUBLASLT_EPILOGUE_BIAS;
      const cudaDataType_t bt = CUDA_R_16BF;
      cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_EPILOGUE, &epi, sizeof(epi));
      cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_BIAS_POINTER, &bias, sizeof(bias));
      cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_BIAS_DATA_TYPE, &bt, sizeof(bt));
    }
    // A = W stored [N, K] row-major = column-major K x N (ld K), used transposed
    if (cublasLtMatrixLayoutCreate(&la, CUDA_R_16BF, K, N, K) != CUBLAS_STATUS_SUCCESS) break;
    // B = X stored [M, K] row-major = column-major K x M (ld K)
    if (cublasLtMatrixLayoutCreate(&lb, CUDA_R_16BF, K, M, K) != CUBLAS_STATUS_SUCCESS) break;
    // C = Y stored [M, N] row-major = column-major N x M (ld N)
    if (cublasLtMatrixLayoutCreate(&lc, CUDA_R_16BF, N, M, N) != CUBLAS_STATUS_SUCCESS) break;
    if (cublasLtMatmulPreferenceCreate(&pref) != CUBLAS_STATUS_SUCCESS) break;
    const size_t ws = kLtWorkspace;
    cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws,
                                         sizeof(ws));
    cublasLtMatmulHeuristicResult_t res;
    int found = 0;
    if (cublasLtMatmulAlgoGetHeuristic(h, op, la, lb, lc, lc, pref, 1, &res, &found) !=
            CUBLAS_STATUS_SUCCESS ||
        found == 0)
      break;
    const float alpha = 1.f, beta = 0.f;
    ok = cublasLtMatmul(h, op, &alpha, W, la, X, lb, &beta, Y, lc, Y, lc, &res.algo, lt_ws, ws,
                        stream) == CUBLAS_STATUS_SUCCESS;
  } while (false);
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (lc) cublasLtMatrixLayoutDestroy(lc);
  if (lb) cublasLtMatrixLayoutDestroy(lb);
  if (la) cublasLtMatrixLayoutDestroy(la);
  if (op) cublasLtMatmulDescDestroy(op);
  return ok;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

size_t mha_workspace_bytes(int B, int L, int E) {
  const size_t act = static_cast<size_t>(B) * L * E * 2;  // one [B, L, E] bf16 tensor
  // qkv (3) + context (1), then the cuBLASLt workspace
  return align256(3 * act) + align256(act) + kLtWorkspace;
}

int launch_mha(const MhaArgs& a, void* workspace, cudaStream_t stream, cudaError_t* err,
               int* lt_status) {
  *err = cudaSuccess;
  *lt_status = 0;
  const int d = a.E / a.H;
  const size_t act = static_cast<size_t>(a.B) * a.L * a.E * 2;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* qkv = reinterpret_cast<uint16_t*>(ws);
  ws += align256(3 * act);
  void* ctx = ws;
  ws += align256(act);
  void* lt_ws = ws;

  int device = 0;
  if ((*err = cudaGetDevice(&device)) != cudaSuccess) return ATTN_ERR_CUDA;
  cublasStatus_t cst;
  cublasLtHandle_t h = lt_handle(device, &cst);
  if (h == nullptr) {
    *lt_status = static_cast<int>(cst);
    return ATTN_ERR_CUDA;
  }
  const int M = a.B * a.L;
  if (!linear_bf16(h, a.x, a.w_qkv, a.b_qkv, qkv, M, 3 * a.E, a.E, lt_ws, stream)) {
    *lt_status = 1;
    return ATTN_ERR_CUDA;
  }
  // q, k, v: the three E-wide thirds of each qkv row, head h at columns h d
  FwdArgs f;
  f.q = qkv;
  f.k = qkv + a.E;
  f.v = qkv + 2 * a.E;
  f.out = ctx;
  f.lse = nullptr;
  f.B = a.B;
  f.H = a.H;
  f.L = a.L;
  f.d = d;
  f.scale = a.scale;
  f.mask_kind = a.mask_kind;
  f.window = a.window;
  f.block_n = 128;
  f.timeout_ns = a.timeout_ns;
  const long long E3 = 3LL * a.E;
  for (int x = 0; x < 3; ++x) {
    f.stride[x][0] = E3;
    f.stride[x][1] = d;
    f.stride[x][2] = E3 * a.L;
  }
  f.stride[3][0] = a.E;  // context [B, L, H, d]
  f.stride[3][1] = d;
  f.stride[3][2] = static_cast<long long>(a.E) * a.L;
  const int st = launch_fwd_bf16_sm100(f, stream, err);
  if (st != ATTN_OK) return st;
  if (!linear_bf16(h, ctx, a.w_out, a.b_out, a.y, M, a.E, a.E, lt_ws, stream)) {
    *lt_status = 2;
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // namespace ebh
