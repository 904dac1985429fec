// sqa_block.cuh -- the parts of one SQAT-m decoder block around the SQA layer
// that are not matrix products: RMS normalisation and its backward (the
// products, including the SwiGLU epilogues and the residual adds, are
// sqa_gemm.cuh's).  SQAT-m model card, "Architecture details": RMS Norm,
// SwiGLU feed-forward of hidden width 768; the block is read as pre-norm with
// residuals, h = x + SQA(RMSNorm(x; g1)), y = h + FFN(RMSNorm(h; g2)).
//
// One warp per row of d elements (d a multiple of 8), 16-byte loads; rows are
// bf16, statistics fp32.
#pragma once

#include "sqa_device.cuh"

namespace sqa {

constexpr float kRmsEps = 1e-6f;

// n = bf16(x * r * g) with r = 1 / sqrt(mean_j x_j^2 + eps); rstd[m] = r.
__global__ void __launch_bounds__(256)
    sqa_rmsnorm_kernel(const __nv_bfloat16* x, const __nv_bfloat16* g, __nv_bfloat16* n, float* rstd, int M, int d) {
  const int warps = blockDim.x >> 5, lane = threadIdx.x & 31;
  for (int m = blockIdx.x * warps + (threadIdx.x >> 5); m < M; m += gridDim.x * warps) {
    const __nv_bfloat16* xr = x + static_cast<long long>(m) * d;
    float ss = 0.f;
    for (int c = lane * 8; c < d; c += 256) {
      const uint4 v = *reinterpret_cast<const uint4*>(xr + c);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 f = __bfloat1622float2(h[u]);
        ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = rsqrtf(ss / static_cast<float>(d) + kRmsEps);
    if (lane == 0) rstd[m] = r;
    __nv_bfloat16* nr = n + static_cast<long long>(m) * d;
    for (int c = lane * 8; c < d; c += 256) {
      const uint4 v = *reinterpret_cast<const uint4*>(xr + c);
      const uint4 gv = *reinterpret_cast<const uint4*>(g + c);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
      const __nv_bfloat162* gg = reinterpret_cast<const __nv_bfloat162*>(&gv);
      uint4 o;
      uint32_t* po = &o.x;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 f = __bfloat1622float2(h[u]), w = __bfloat1622float2(gg[u]);
        po[u] = dev::pack_bf16x2(f.x * r * w.x, f.y * r * w.y);
      }
      *reinterpret_cast<uint4*>(nr + c) = o;
    }
  }
}

// Backward of n = x r g for the rows of x, given dn (the gradient of the
// normalised rows) and the saved r:
//   dx = resid + r (dn g) - r^3 x sum_j(dn_j g_j x_j) / d   (bf16)
//   dg += sum_m dn x r                                      (fp32, reduced per
//         block in shared memory, then added to dg: run-dependent order)
// dg must hold zeros (or a partial sum) before the launch; smem: d floats.
__global__ void __launch_bounds__(256)
    sqa_rmsnorm_bwd_kernel(const __nv_bfloat16* x, const __nv_bfloat16* g, const float* rstd,
                           const __nv_bfloat16* dn, const __nv_bfloat16* resid, __nv_bfloat16* dx, float* dg, int M,
                           int d) {
  extern __shared__ float dg_part[];
  for (int j = threadIdx.x; j < d; j += blockDim.x) dg_part[j] = 0.f;
  __syncthreads();
  const int warps = blockDim.x >> 5, lane = threadIdx.x & 31;
  for (int m = blockIdx.x * warps + (threadIdx.x >> 5); m < M; m += gridDim.x * warps) {
    const long long row = static_cast<long long>(m) * d;
    const float r = rstd[m];
    float dot = 0.f;
    for (int c = lane * 8; c < d; c += 256) {
      const uint4 xv = *reinterpret_cast<const uint4*>(x + row + c);
      const uint4 nv = *reinterpret_cast<const uint4*>(dn + row + c);
      const uint4 gv = *reinterpret_cast<const uint4*>(g + c);
      const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xv);
      const __nv_bfloat162* nh = reinterpret_cast<const __nv_bfloat162*>(&nv);
      const __nv_bfloat162* gh = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 xf = __bfloat1622float2(xh[u]), nf = __bfloat1622float2(nh[u]), gf = __bfloat1622float2(gh[u]);
        dot = fmaf(nf.x * gf.x, xf.x, fmaf(nf.y * gf.y, xf.y, dot));
        atomicAdd(&dg_part[c + 2 * u], nf.x * xf.x * r);
        atomicAdd(&dg_part[c + 2 * u + 1], nf.y * xf.y * r);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    const float k = r * r * r * dot / static_cast<float>(d);
    for (int c = lane * 8; c < d; c += 256) {
      const uint4 xv = *reinterpret_cast<const uint4*>(x + row + c);
      const uint4 nv = *reinterpret_cast<const uint4*>(dn + row + c);
      const uint4 gv = *reinterpret_cast<const uint4*>(g + c);
      const uint4 rv = *reinterpret_cast<const uint4*>(resid + row + c);
      const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xv);
      const __nv_bfloat162* nh = reinterpret_cast<const __nv_bfloat162*>(&nv);
      const __nv_bfloat162* gh = reinterpret_cast<const __nv_bfloat162*>(&gv);
      const __nv_bfloat162* rh = reinterpret_cast<const __nv_bfloat162*>(&rv);
      uint4 o;
      uint32_t* po = &o.x;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 xf = __bfloat1622float2(xh[u]), nf = __bfloat1622float2(nh[u]), gf = __bfloat1622float2(gh[u]);
        const float2 rf = __bfloat1622float2(rh[u]);
        po[u] = dev::pack_bf16x2(rf.x + r * nf.x * gf.x - k * xf.x, rf.y + r * nf.y * gf.y - k * xf.y);
      }
      *reinterpret_cast<uint4*>(dx + row + c) = o;
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < d; j += blockDim.x) atomicAdd(&dg[j], dg_part[j]);
}

}  // namespace sqa
