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

// ---------------------------------------------------------------- FP8 latent KV rows
// Block-wise KV cache write (Block-Wise Quantization for Key-Value Cache,
// section 4 of "Optimizing Inference for New Model Architectures ..."; the
// Tiered Quantization table of "Day-0 Inference Adaptation ..."): per token,
// the DC latent dims in tiles of min(128, DC) elements, each with the same
// per-group rule as the index keys; the DR rope dims stay bf16. One packed
// row per token (ROW_BYTES, a multiple of 16):
//   [0, DC)                 E4M3 codes of the latent dims
//   [DC, DC + 2 DR)         the rope dims, bf16
//   [DC + 2 DR, + 4 NT)     the NT tile scales, fp32
//   zero padding up to ROW_BYTES
template <int DC, int DR>
struct KvFp8Row {
  static constexpr int TILE = DC < 128 ? DC : 128;
  static constexpr int NT = DC / TILE;
  static constexpr int ROPE_OFF = DC;
  static constexpr int SCALE_OFF = DC + 2 * DR;
  static constexpr int ROW_BYTES = ((SCALE_OFF + 4 * NT + 15) / 16) * 16;
  static_assert(DC % TILE == 0 && DC % 64 == 0 && DR % 8 == 0, "latent / rope dims");
};

// One warp per row; lane l owns elements [4l, 4l+4) of each 128-element
// slice (as in quantize_keys_kernel), lanes 0..DR/8-1 copy the rope dims.
template <int DC, int DR>
__global__ void __launch_bounds__(256) quantize_kv_kernel(const __nv_bfloat16* __restrict__ kv, int64_t n_rows,
                                                          uint8_t* __restrict__ out) {
  using R = KvFp8Row<DC, DR>;
  constexpr int D = DC + DR;
  constexpr int LANES_PER_TILE = R::TILE / 4;
  const int warps_per_block = blockDim.x >> 5;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * warps_per_block + warp_id();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * warps_per_block;
  const int lane = lane_id();
  for (int64_t row = first; row < n_rows; row += stride) {
    const __nv_bfloat16* src = kv + row * D;
    uint8_t* dst = out + row * R::ROW_BYTES;
#pragma unroll
    for (int base = 0; base < DC; base += 128) {
      const int e = base + lane * 4;
      const bool active = e < DC;
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      if (active) {
        const uint2 raw = *reinterpret_cast<const uint2*>(src + e);
        const __nv_bfloat162 p0 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
        const __nv_bfloat162 p1 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
        x[0] = __low2float(p0);
        x[1] = __high2float(p0);
        x[2] = __low2float(p1);
        x[3] = __high2float(p1);
      }
      float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
      for (int off = LANES_PER_TILE / 2; off >= 1; off >>= 1)
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const float s = __fdiv_rn(amax, 448.0f);
      if (active) {
        uint32_t codes = 0u;
        if (s != 0.0f)
          codes = e4m3x4_from_f32(__fdiv_rn(x[0], s), __fdiv_rn(x[1], s), __fdiv_rn(x[2], s),
                                  __fdiv_rn(x[3], s));
        *reinterpret_cast<uint32_t*>(dst + e) = codes;
        if ((lane % LANES_PER_TILE) == 0) *reinterpret_cast<float*>(dst + R::SCALE_OFF + 4 * (e / R::TILE)) = s;
      }
    }
    // rope dims (16-byte chunks) and the zero padding after the scales
    if (lane < DR / 8)
      *reinterpret_cast<uint4*>(dst + R::ROPE_OFF + 16 * lane) = *reinterpret_cast<const uint4*>(src + DC + 8 * lane);
    for (int o = R::SCALE_OFF + 4 * R::NT + 4 * lane; o < R::ROW_BYTES; o += 128)
      *reinterpret_cast<uint32_t*>(dst + o) = 0u;
  }
}

// ---------------------------------------------------------------- MXFP8 (index queries and keys)
// Index Q/K Uses MXFP8 (section 4.2 of "Inference Adaptation and Performance
// Optimization for New Large Language Model Architectures"): 32 elements
// share one scale. The scale is absmax / 448 rounded up to a power of two,
// 2^e with e the least integer such that 448 * 2^e >= absmax, kept in
// [-127, 127] and stored as the E8M0 byte e + 127 (absmax 0: e = -127,
// codes 0). From the fp32 bits of absmax = m 2^E (1 <= m < 2):
// e = E - 8, plus 1 when m > 1.75 (448 = 1.75 * 2^8). Codes: the E4M3 cast
// (nearest even, saturating) of x * 2^-e, a product that is exact.
__device__ __forceinline__ int mx_exponent(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  const int E = static_cast<int>((bits >> 23) & 0xFFu);
  if (E == 0) return -127;  // zero or below the normal range
  int e = E - 127 - 8 + ((bits & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^k as fp32 for k in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float exp2_int(int k) {
  return k >= -126 ? __uint_as_float(static_cast<uint32_t>(k + 127) << 23) : __uint_as_float(0x00400000u);
}

// One warp per row of `dim` (a multiple of 32, <= 1024) elements; lane l
// owns elements [4l, 4l+4) of each 128-element slice (8 lanes per group).
__global__ void __launch_bounds__(256) mx_quantize_kernel(const __nv_bfloat16* __restrict__ x, int64_t n_rows,
                                                          int dim, uint8_t* __restrict__ codes,
                                                          uint8_t* __restrict__ scales) {
  const int warps_per_block = blockDim.x >> 5;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * warps_per_block + warp_id();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * warps_per_block;
  const int lane = lane_id();
  for (int64_t row = first; row < n_rows; row += stride) {
    for (int base = 0; base < dim; base += 128) {
      const int e0 = base + lane * 4;
      const bool active = e0 < dim;
      float v[4] = {0.f, 0.f, 0.f, 0.f};
      if (active) {
        const uint2 raw = *reinterpret_cast<const uint2*>(x + row * dim + e0);
        const __nv_bfloat162 p0 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
        const __nv_bfloat162 p1 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
        v[0] = __low2float(p0);
        v[1] = __high2float(p0);
        v[2] = __low2float(p1);
        v[3] = __high2float(p1);
      }
      float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
      for (int off = 4; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      const int e = mx_exponent(amax);
      if (active) {
        const float m = exp2_int(-e);
        *reinterpret_cast<uint32_t*>(codes + row * dim + e0) = e4m3x4_from_f32(v[0] * m, v[1] * m, v[2] * m, v[3] * m);
        if ((lane & 7) == 0) scales[row * (dim / 32) + e0 / 32] = static_cast<uint8_t>(e + 127);
      }
    }
  }
}

// codes [n] with one E8M0 byte per 32 -> bf16 [n] (exact while the value stays
// inside bf16's normal range).
__global__ void __launch_bounds__(256) mx_dequantize_kernel(const uint8_t* __restrict__ codes,
                                                            const uint8_t* __restrict__ scales, int64_t n,
                                                            __nv_bfloat16* __restrict__ out) {
  const int64_t n4 = n / 4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e = i * 4;
    const uint32_t c = *reinterpret_cast<const uint32_t*>(codes + e);
    const float m = exp2_int(static_cast<int>(scales[e / 32]) - 127);
    const __half2_raw h01 = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(c & 0xFFFFu), __NV_E4M3);
    const __half2_raw h23 = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(c >> 16), __NV_E4M3);
    float2 a = __half22float2(__half2(h01)), b = __half22float2(__half2(h23));
    const __nv_bfloat162 b01 = __float22bfloat162_rn(make_float2(a.x * m, a.y * m));
    const __nv_bfloat162 b23 = __float22bfloat162_rn(make_float2(b.x * m, b.y * m));
    uint2 o;
    o.x = *reinterpret_cast<const uint32_t*>(&b01);
    o.y = *reinterpret_cast<const uint32_t*>(&b23);
    *reinterpret_cast<uint2*>(out + e) = o;
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
