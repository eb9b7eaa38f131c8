// quant.cuh -- index-key cache write: per-group dynamic FP8 (E4M3)
// quantisation and its inverse.
//
// Follows the per-group scheme of the Tiered Quantization table and its
// pseudocode in "Day-0 Inference Adaptation and Performance Optimization for
// New-Architecture Large Language Models": scale = max|group| / quant_max,
// then the 8-bit cast; quant_max = 448 (largest finite E4M3). Precisely:
//   s = fl32(absmax / 448);  s == 0 -> codes 0;
//   code = e4m3(round-to-nearest-even, saturate to +-448)(fl32(k / s)).
// Both divisions are IEEE round-to-nearest (no fast math in this build).
//
// Layout: one warp per key row; lane l owns elements [4l, 4l+4) of each
// 128-element slice, so a group of G elements spans G/4 lanes and its absmax
// is a shuffle reduction inside that lane segment. Loads are 8-byte bf16x4,
// stores 4-byte fp8x4: fully coalesced, HBM-bound.
#pragma once
#include "dsa_common.cuh"

namespace dsa {

__device__ __forceinline__ uint32_t e4m3x4_from_f32(float a, float b, float c, float d) {
  const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

template <int GROUP>
__global__ void __launch_bounds__(256) quantize_keys_kernel(const __nv_bfloat16* __restrict__ k, int64_t n_keys,
                                                            int dim, uint8_t* __restrict__ k8,
                                                            float* __restrict__ scale) {
  constexpr int LANES_PER_GROUP = GROUP / 4;
  const int warps_per_block = blockDim.x >> 5;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * warps_per_block + warp_id();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * warps_per_block;
  const int lane = lane_id();
  const int groups_per_row = dim / GROUP;
  for (int64_t row = first; row < n_keys; row += stride) {
    for (int base = 0; base < dim; base += 128) {
      const int e = base + lane * 4;
      const bool active = e < dim;
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      if (active) {
        const uint2 raw = *reinterpret_cast<const uint2*>(k + row * dim + e);
        const __nv_bfloat162 p0 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
        const __nv_bfloat162 p1 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
        x[0] = __low2float(p0);
        x[1] = __high2float(p0);
        x[2] = __low2float(p1);
        x[3] = __high2float(p1);
      }
      float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
      for (int off = LANES_PER_GROUP / 2; off >= 1; off >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const float s = __fdiv_rn(amax, 448.0f);
      if (active) {
        uint32_t codes = 0u;
        if (s != 0.0f)
          codes = e4m3x4_from_f32(__fdiv_rn(x[0], s), __fdiv_rn(x[1], s), __fdiv_rn(x[2], s),
                                  __fdiv_rn(x[3], s));
        *reinterpret_cast<uint32_t*>(k8 + row * dim + e) = codes;
        if ((lane % LANES_PER_GROUP) == 0) scale[row * groups_per_row + e / GROUP] = s;
      }
    }
  }
}

__global__ void __launch_bounds__(256) dequantize_keys_kernel(const uint8_t* __restrict__ k8,
                                                              const float* __restrict__ scale, int64_t n,
                                                              int dim, int group, float* __restrict__ out) {
  const int64_t n4 = n / 4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = i * 4;
    const int64_t row = e / dim;
    const int col = static_cast<int>(e - row * dim);
    const uint32_t c = *reinterpret_cast<const uint32_t*>(k8 + e);
    const float s = scale[row * (dim / group) + col / group];  // 4 | group: one scale
    float4 o;
    o.x = __half2float(__half(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c & 0xFF), __NV_E4M3))) * s;
    o.y = __half2float(__half(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>((c >> 8) & 0xFF), __NV_E4M3))) * s;
    o.z = __half2float(__half(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>((c >> 16) & 0xFF), __NV_E4M3))) * s;
    o.w = __half2float(__half(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c >> 24), __NV_E4M3))) * s;
    *reinterpret_cast<float4*>(out + e) = o;
  }
}

}  // namespace dsa
