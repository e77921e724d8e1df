// attn_merge.cu -- exact merge of attention partials computed over disjoint
// key ranges (split-KV on one GPU, or key shards on several).
//
// A partial over keys K_s gives O_s = sum_{j in K_s} e^{s_ij - LSE_s} v_j and
// LSE_s = ln sum_{j in K_s} e^{s_ij}.  Over the union of the ranges,
//     LSE = ln sum_s e^{LSE_s},   O = sum_s e^{LSE_s - LSE} O_s,
// the combination step the page "Mosaic multi-GPU sequence-sharded attention"
// (kwkr.cn), section 2.1, calls the tree reduction of local attention results.
// Splits whose key range holds no allowed key of a row are skipped for that
// row (they were never written for it).  Rows may sit at an offset into the
// keys (a rank's rows of a sequence-sharded problem).  One warp per row; each lane owns
// d/32 consecutive columns, read as one vector.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "attn.h"
#include "kernels.h"
#include "tiles.h"

namespace ebh {
namespace {

constexpr int kMergeWarps = 8;

template <int D>
__global__ void __launch_bounds__(kMergeWarps * 32) attn_merge_kernel(const MergeArgs m) {
  // in a dependent launch: the partials' writer has completed from here on
  // (a no-op otherwise)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  constexpr int E = D / 32;  // columns per lane
  const long long row = static_cast<long long>(blockIdx.x) * kMergeWarps + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= static_cast<long long>(m.BH) * m.L) return;
  const int bh = static_cast<int>(row / m.L);
  const int i = static_cast<int>(row % m.L);

  // allowed keys of row i (key position qp): [kmin, kmax]
  const long long qp = static_cast<long long>(m.q_offset) + i;
  long long kmin = 0, kmax = static_cast<long long>(m.kv_len) - 1;
  if (m.mask_kind == kMaskCausal) {
    kmax = qp < kmax ? qp : kmax;
  } else if (m.mask_kind == kMaskWindow) {
    kmin = qp - m.window > 0 ? qp - m.window : 0;
    kmax = qp + m.window < kmax ? qp + m.window : kmax;
  } else if (m.mask_kind == kMaskCausalWindow) {
    kmin = qp - m.window > 0 ? qp - m.window : 0;
    kmax = qp < kmax ? qp : kmax;
  }
  auto contributes = [&](int s) {
    const long long lo = m.bounds[s] > kmin ? m.bounds[s] : kmin;
    const long long hi = (long long)m.bounds[s + 1] - 1 < kmax ? m.bounds[s + 1] - 1 : kmax;
    return lo <= hi;
  };

  float mx = -INFINITY;
  for (int s = 0; s < m.num_splits; ++s)
    if (contributes(s))
      mx = fmaxf(mx, m.lse_part[(static_cast<size_t>(s) * m.BH + bh) * m.L + i]);

  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float sum = 0.f;
  if (mx != -INFINITY) {
    for (int s = 0; s < m.num_splits; ++s) {
      if (!contributes(s)) continue;
      const size_t head = static_cast<size_t>(s) * m.BH + bh;
      const float w = expf(m.lse_part[head * m.L + i] - mx);
      sum += w;
      const float* src = m.o_part + (head * m.L + i) * D + lane * E;
      if constexpr (E == 4) {
        const float4 v = *reinterpret_cast<const float4*>(src);
        acc[0] = fmaf(w, v.x, acc[0]);
        acc[1] = fmaf(w, v.y, acc[1]);
        acc[2] = fmaf(w, v.z, acc[2]);
        acc[3] = fmaf(w, v.w, acc[3]);
      } else {
        const float2 v = *reinterpret_cast<const float2*>(src);
        acc[0] = fmaf(w, v.x, acc[0]);
        acc[1] = fmaf(w, v.y, acc[1]);
      }
    }
  }
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  const size_t dst = (static_cast<size_t>(bh) * m.L + i) * D + lane * E;
  if (m.out_f32) {
    float* o = static_cast<float*>(m.out) + dst;
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] = acc[e] * inv;
  } else {
    uint32_t pk[E / 2];
#pragma unroll
    for (int e = 0; e < E / 2; ++e) {
      uint32_t r;
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(acc[2 * e + 1] * inv), "f"(acc[2 * e] * inv));
      pk[e] = r;
    }
    uint16_t* o = static_cast<uint16_t*>(m.out) + dst;
    if constexpr (E == 4) {
      *reinterpret_cast<uint2*>(o) = make_uint2(pk[0], pk[1]);
    } else {
      *reinterpret_cast<uint32_t*>(o) = pk[0];
    }
  }
  if (lane == 0 && m.lse != nullptr)
    m.lse[static_cast<size_t>(bh) * m.L + i] = sum > 0.f ? mx + logf(sum) : -INFINITY;
}

}  // namespace

int launch_merge(const MergeArgs& m, cudaStream_t stream, cudaError_t* err) {
  *err = cudaSuccess;
  const long long rows = static_cast<long long>(m.BH) * m.L;
  const long long blocks = (rows + kMergeWarps - 1) / kMergeWarps;
  if (blocks > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (m.d != 128 && m.d != 64) return ATTN_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(kMergeWarps * 32);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = m.dependent ? 1 : 0;
  *err = m.d == 128 ? cudaLaunchKernelEx(&cfg, attn_merge_kernel<128>, m)
                    : cudaLaunchKernelEx(&cfg, attn_merge_kernel<64>, m);
  return *err == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace ebh
