// Shared device-side definitions of the ZHA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zha.h"

namespace zha {

constexpr int kMaxLevels = 20;   // b >= 2 and capacity < 2^31 keep L well below this
constexpr int kMaxRefs = 32;
constexpr int kMaxDevices = 128;  // CUDA devices a process can address (per-device state of the library)

// ---------------------------------------------------------------- element types
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Elements of type T in one 16-byte vector.
template <typename T> struct Vec { static constexpr int N = 16 / sizeof(T); };

// Read-only 16-byte global load (no L1 allocation: the cache lines are streamed).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Unpack a 16-byte vector of T into fp32.
template <typename T> __device__ __forceinline__ void unpack16(const uint4& v, float* out);
template <> __device__ __forceinline__ void unpack16<float>(const uint4& v, float* out) {
  out[0] = __uint_as_float(v.x);
  out[1] = __uint_as_float(v.y);
  out[2] = __uint_as_float(v.z);
  out[3] = __uint_as_float(v.w);
}
template <> __device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4& v, float* out) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    out[2 * i] = __uint_as_float(w[i] << 16);          // low half: element 2i
    out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);  // high half: element 2i+1
  }
}

// D (16x8, fp32) += A (16x16, bf16, row) x B (16x8, bf16, col), one warp.
__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void mma_f16_16816(float* c, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// ---------------------------------------------------------------- FP4 router planes
// Values of the e2m1 codes by magnitude index 0..7 (the code's low three bits; bit 3 is the sign).
// A group of 16 slopes shares one e4m3 scale; the slope is code * scale (see zha.h, ZHA_PLANES_FP4).

// Nearest e4m3 value of x >= 0, ties to the even mantissa, at most 448 (the largest finite e4m3);
// *bits receives its encoding (sign 0, exponent bias 7, 3 mantissa bits).  Scaling by powers of two
// and rintf (round half to even) are exact, so the result is the correctly rounded one.
__device__ __forceinline__ float e4m3_nearest(float x, uint32_t* bits) {
  if (!(x > 0.f)) {
    *bits = 0u;
    return 0.f;
  }
  if (x >= 448.f) {
    *bits = 0x7Eu;
    return 448.f;
  }
  int e2;
  frexpf(x, &e2);
  int E = e2 - 1;  // x in [2^E, 2^(E+1))
  if (E < -6) {    // subnormal range: multiples of 2^-9
    const float m = rintf(ldexpf(x, 9));
    *bits = uint32_t(m);  // m == 8 is the smallest normal (exponent field 1, mantissa 0)
    return ldexpf(m, -9);
  }
  float m = rintf(ldexpf(x, 3 - E));  // in [8, 16]
  if (m == 16.f) {
    m = 8.f;
    ++E;
  }
  const float v = ldexpf(m, E - 3);
  if (v > 448.f) {
    *bits = 0x7Eu;
    return 448.f;
  }
  *bits = (uint32_t(E + 7) << 3) | (uint32_t(m) - 8u);
  return v;
}

// e2m1 code of y: nearest of {0, 0.5, 1, 1.5, 2, 3, 4, 6} with the sign of y, ties to the even
// mantissa, at most 6; magnitude 0 is coded +0.
__device__ __forceinline__ uint32_t e2m1_code(float y) {
  const float a = fabsf(y);
  uint32_t i;
  if (a <= 0.25f) i = 0u;
  else if (a < 0.75f) i = 1u;
  else if (a <= 1.25f) i = 2u;
  else if (a < 1.75f) i = 3u;
  else if (a <= 2.5f) i = 4u;
  else if (a < 3.5f) i = 5u;
  else if (a <= 5.f) i = 6u;
  else i = 7u;
  return i == 0u ? 0u : (i | (y < 0.f ? 8u : 0u));
}

// Two e2m1 codes (low nibble first) -> f16x2 (low half first), exact.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte2) {
  uint32_t r;
  asm("{\n .reg .b8 lo8, hi8;\n mov.b16 {lo8, hi8}, %1;\n cvt.rn.f16x2.e2m1x2 %0, lo8;\n}"
      : "=r"(r)
      : "h"((unsigned short)(byte2 & 0xffu)));
  return r;
}

// Two e4m3 values (low byte first) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"((unsigned short)(two & 0xffffu)));
  return r;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int w) {
  return w == 0 ? v.x : (w == 1 ? v.y : (w == 2 ? v.z : v.w));
}

// ---------------------------------------------------------------- ordered keys
// Order-preserving map of fp32 onto uint32 (ascending), and the descending key
// used to rank routing candidates: a smaller key means a larger estimate.
__device__ __forceinline__ uint32_t float_to_ordered(float x) {
  uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ordered_to_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}
__device__ __forceinline__ uint32_t desc_key(float e) { return ~float_to_ordered(e); }
__device__ __forceinline__ float desc_key_value(uint32_t k) { return ordered_to_float(~k); }

// Node codes: level in the top 5 bits, index within the level in the low 27.
__device__ __forceinline__ uint32_t node_code(int level, uint32_t idx) {
  return (uint32_t(level) << 27) | idx;
}
__device__ __forceinline__ int code_level(uint32_t c) { return int(c >> 27); }
__device__ __forceinline__ uint32_t code_index(uint32_t c) { return c & 0x07ffffffu; }

// ---------------------------------------------------------------- tree description
// Everything a kernel needs to address the node storage of one tree.
struct TreeDev {
  int d, hq, hkv, group, block, levels, refs, chunk_level;
  int64_t capacity;
  int64_t cap_nodes[kMaxLevels + 1];   // node slots per KV head per level
  int64_t pow_b[kMaxLevels + 1];       // block^level (tokens per node)
  uint64_t rec_off[kMaxLevels + 1];    // byte offsets in the node buffer
  uint64_t f_off[kMaxLevels + 1];
  uint64_t up_off[kMaxLevels + 1];     // fp32 full nodes, levels chunk_level .. levels-1
  uint64_t rec_bytes;                  // mu[R][d] (element type) + bias[R] fp32, padded to 16 B
  uint64_t up_bytes;                   // mu[R][d] fp32 + f[R] + g[R]
  int planes;                          // ZHA_PLANES_KEY or ZHA_PLANES_FP4 (the routing steps read rec4)
  uint64_t rec4_off[kMaxLevels + 1];   // FP4 router records: codes[R][d/2], scales[R][d/16], bias[R]
  uint64_t rec4_bytes;
  char* nodes;
  void* K;
  void* V;
  const void* refsp;
  int* status;
  float inv_sqrt_d;

  __device__ __forceinline__ char* rec(int level, int head, int64_t i) const {
    return nodes + rec_off[level] + (uint64_t(head) * cap_nodes[level] + i) * rec_bytes;
  }
  __device__ __forceinline__ char* rec4(int level, int head, int64_t i) const {
    return nodes + rec4_off[level] + (uint64_t(head) * cap_nodes[level] + i) * rec4_bytes;
  }
  __device__ __forceinline__ float* fval(int level, int head, int64_t i) const {
    return reinterpret_cast<float*>(nodes + f_off[level]) +
           (uint64_t(head) * cap_nodes[level] + i) * refs;
  }
  __device__ __forceinline__ float* up(int level, int head, int64_t i) const {
    return reinterpret_cast<float*>(nodes + up_off[level] + (uint64_t(head) * cap_nodes[level] + i) * up_bytes);
  }
};

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

__device__ __forceinline__ void raise_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

}  // namespace zha
