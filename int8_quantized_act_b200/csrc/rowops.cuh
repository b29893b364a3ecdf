// rowops.cuh - device helpers shared by the row kernels: 8-wide vector loads
// and stores of float32 / bf16, the block-Hadamard butterflies of one
// 256-element chunk held by a warp, and warp reductions.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace ql {

// -------------------------------------------------------------- 8-wide I/O
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// bf16 -> float32 is exact: the bf16 bits are the top half of the float.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
  const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return a | (b << 16);
}

__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
  *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                            pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

// -------------------------------------------------------------- int8 codes
// Round to nearest even, clamp to [-127, 127].
__device__ __forceinline__ int code_rne(float t) {
  float r = rintf(t);
  r = fminf(fmaxf(r, -127.0f), 127.0f);
  return static_cast<int>(r);
}

// Round-to-nearest-even of v through the float adder, for |v| <= 127.5:
// v + 1.5*2^23 lies in [2^23, 2^24), where adjacent floats are 1 apart, so
// the IEEE addition itself rounds v to an integer, ties to even (exactly
// rintf(v)).  The integer sits in the low mantissa bits of the sum: its low
// byte is the int8 code.  Callers guarantee |v| <= 127(1 + 2^-22) (v = t *
// 127/amax with |t| <= amax); for inf/NaN inputs the byte is unspecified,
// like every output under QL_ERR_NONFINITE.
constexpr float kRneMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ uint32_t rne_bits(float v) { return __float_as_uint(__fadd_rn(v, kRneMagic)); }

// rne_bits(t * f) with the product rounded first: __fmul_rn / __fadd_rn are
// never merged into a fused multiply-add, which would skip the product's
// rounding and break exact ties (t * f = k + 1/2) differently.
__device__ __forceinline__ uint32_t rne_bits_prod(float t, float f) {
  return __float_as_uint(__fadd_rn(__fmul_rn(t, f), kRneMagic));
}

// Low bytes of four rne_bits words, packed little-endian.
__device__ __forceinline__ uint32_t pack_codes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Running max of |x| kept as the bit pattern of a non-negative float: for
// finite values the integer order is the float order; inf and NaN patterns
// (>= 0x7F800000) sort above every finite value, so one compare at the end
// tells whether a non-finite value was met.
__device__ __forceinline__ uint32_t abs_bits(float x) { return __float_as_uint(x) & 0x7FFFFFFFu; }

constexpr uint32_t kInfBits = 0x7F800000u;

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  return (static_cast<uint32_t>(a) & 0xFFu) | ((static_cast<uint32_t>(b) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(c) & 0xFFu) << 16) | ((static_cast<uint32_t>(d) & 0xFFu) << 24);
}

// -------------------------------------------------------------- packed pairs
// sm_100a executes two float32 additions / multiplications per instruction
// (add/sub/mul.rn.f32x2); each half is an ordinary IEEE round-to-nearest
// operation, so results are bit-identical to the scalar forms.  A packed
// multiply whose result feeds a packed add can be compiled into a fused
// multiply-add (observed on this toolchain even with -fmad=false), so the
// packed forms are used only where no product is added afterwards: the
// butterflies (additions only) and the rotation's final scaling.
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// a * b + c for two pairs (fma.rn.f32x2), each rounded once.  Used only with
// b = +-1, where the product is exact: fma(own, +-1, p) = p +- own rounded
// once, the same bits as the butterfly's addition or subtraction.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// v[i] = v[i] * c for 8 values, two per instruction.
__device__ __forceinline__ void scale8(float (&v)[8], float c) {
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 r = mul2(make_float2(v[i], v[i + 1]), make_float2(c, c));
    v[i] = r.x;
    v[i + 1] = r.y;
  }
}

// Codes of 8 values: rne(v[i] * inv) through the adder (see rne_bits_prod).
__device__ __forceinline__ uint2 codes8(const float (&v)[8], float inv) {
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) b[i] = rne_bits_prod(v[i], inv);
  return make_uint2(pack_codes(b[0], b[1], b[2], b[3]), pack_codes(b[4], b[5], b[6], b[7]));
}

// -------------------------------------------------------------- Hadamard
// The butterflies of fwht_chunk with the block size fixed at compile time
// (HB = 2..256) and the additions done two at a time.  Same operations in
// the same order as fwht_chunk, so the same bits.
template <int HB>
__device__ __forceinline__ void fwht_chunk_ct(float (&v)[8], int lane, float c) {
  if constexpr (HB >= 2) {  // h = 1: pairs (0,1) (2,3) (4,5) (6,7)
    const float2 a0 = make_float2(v[0], v[2]), b0 = make_float2(v[1], v[3]);
    const float2 a1 = make_float2(v[4], v[6]), b1 = make_float2(v[5], v[7]);
    const float2 s0 = add2(a0, b0), d0 = sub2(a0, b0), s1 = add2(a1, b1), d1 = sub2(a1, b1);
    v[0] = s0.x; v[1] = d0.x; v[2] = s0.y; v[3] = d0.y;
    v[4] = s1.x; v[5] = d1.x; v[6] = s1.y; v[7] = d1.y;
  }
  if constexpr (HB >= 4) {  // h = 2: pairs (0,2) (1,3) (4,6) (5,7)
    const float2 a0 = make_float2(v[0], v[1]), b0 = make_float2(v[2], v[3]);
    const float2 a1 = make_float2(v[4], v[5]), b1 = make_float2(v[6], v[7]);
    const float2 s0 = add2(a0, b0), d0 = sub2(a0, b0), s1 = add2(a1, b1), d1 = sub2(a1, b1);
    v[0] = s0.x; v[1] = s0.y; v[2] = d0.x; v[3] = d0.y;
    v[4] = s1.x; v[5] = s1.y; v[6] = d1.x; v[7] = d1.y;
  }
  if constexpr (HB >= 8) {  // h = 4: pairs (0,4) (1,5) (2,6) (3,7)
    const float2 a0 = make_float2(v[0], v[1]), b0 = make_float2(v[4], v[5]);
    const float2 a1 = make_float2(v[2], v[3]), b1 = make_float2(v[6], v[7]);
    const float2 s0 = add2(a0, b0), d0 = sub2(a0, b0), s1 = add2(a1, b1), d1 = sub2(a1, b1);
    v[0] = s0.x; v[1] = s0.y; v[4] = d0.x; v[5] = d0.y;
    v[2] = s1.x; v[3] = s1.y; v[6] = d1.x; v[7] = d1.y;
  }
#pragma unroll
  for (int h = 8; h < HB; h <<= 1) {
    const int d = h >> 3;
    const uint32_t flip = (lane & d) ? 0x80000000u : 0u;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const float p0 = __shfl_xor_sync(0xFFFFFFFFu, v[i], d);
      const float p1 = __shfl_xor_sync(0xFFFFFFFFu, v[i + 1], d);
      const float2 r = add2(make_float2(p0, p1),
                            make_float2(__uint_as_float(__float_as_uint(v[i]) ^ flip),
                                        __uint_as_float(__float_as_uint(v[i + 1]) ^ flip)));
      v[i] = r.x;
      v[i + 1] = r.y;
    }
  }
  scale8(v, c);
}

// Block-Hadamard rotation of one 256-element chunk spread across a warp,
// lane l holding elements 8l..8l+7 in v.  For blocks of B elements (B a power
// of two, 2..256) the Sylvester butterflies run for h = 1, 2, ..., B/2 in that
// order, pair (j, j+h) -> (v_j + v_{j+h}, v_j - v_{j+h}); stages with h < 8
// stay inside a lane, larger h exchange with lane ^ (h/8).  Then every value
// is multiplied by c = fl32(1/sqrt(B)).  All 32 lanes must call this.
__device__ __forceinline__ void fwht_chunk(float (&v)[8], int B, int lane, float c) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
    if (h < B) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if ((i & h) == 0) {
          const float a = v[i], b = v[i + h];
          v[i] = a + b;
          v[i + h] = a - b;
        }
      }
    }
  }
  for (int h = 8; h < B; h <<= 1) {
    const int d = h >> 3;
    // The lane holding the higher index computes partner - own = partner +
    // (-own): flip the sign bit instead of selecting between two sums.
    const uint32_t flip = (lane & d) ? 0x80000000u : 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float p = __shfl_xor_sync(0xFFFFFFFFu, v[i], d);
      v[i] = p + __uint_as_float(__float_as_uint(v[i]) ^ flip);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = v[i] * c;
}

// Block-128 rotation of a 1024-column chunk spread across a warp, lane l
// holding columns 32l .. 32l+31 (lanes 4b .. 4b+3 hold block b): the
// butterflies h = 1..16 stay inside the lane, h = 32 and 64 pair lanes l^1
// and l^2 (the higher index takes partner - own), then every value is
// multiplied by c.  The same operations in the same order as fwht_chunk with
// B = 128, so the same bits, with half the shuffles.
__device__ __forceinline__ void fwht128_wide(float (&v)[32], int lane, float c) {
  // h = 1: pairs (i, i+1), one scalar add and subtract each (the pair's two
  // halves would need to be regrouped for a packed operation); the later
  // stages combine the register pairs (i, i+1) and (i+h, i+h+1) as they are.
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float a = v[i], b = v[i + 1];
    v[i] = a + b;
    v[i + 1] = a - b;
  }
#pragma unroll
  for (int h = 2; h < 32; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      if ((i & h) == 0) {  // pairs (i, i+h), (i+1, i+1+h)
        const float2 a = make_float2(v[i], v[i + 1]), b = make_float2(v[i + h], v[i + h + 1]);
        const float2 s2 = add2(a, b), d2 = sub2(a, b);
        v[i] = s2.x; v[i + 1] = s2.y; v[i + h] = d2.x; v[i + h + 1] = d2.y;
      }
    }
  }
#pragma unroll
  for (int d = 1; d <= 2; d <<= 1) {
    const float sg = (lane & d) ? -1.0f : 1.0f;
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const float p0 = __shfl_xor_sync(0xFFFFFFFFu, v[i], d);
      const float p1 = __shfl_xor_sync(0xFFFFFFFFu, v[i + 1], d);
      const float2 r = fma2(make_float2(v[i], v[i + 1]), make_float2(sg, sg), make_float2(p0, p1));
      v[i] = r.x;
      v[i + 1] = r.y;
    }
  }
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float2 r = mul2(make_float2(v[i], v[i + 1]), make_float2(c, c));
    v[i] = r.x;
    v[i + 1] = r.y;
  }
}

// -------------------------------------------------------------- NaN-aware maxima
// max(a, b) that is NaN whenever an operand is NaN (max.NaN.f32), where
// fmaxf would drop the NaN.  With |x| operands the running maximum of a row
// or column is then NaN as soon as one element is NaN and +inf when one is
// infinite, so a single compare of its bit pattern against kInfBits tells
// whether a non-finite value was met.
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// The three-operand form (sm_100): max(a, b, c), NaN if any operand is NaN.
__device__ __forceinline__ float fmax3_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// The NaN-propagating minima (min.NaN.f32, two and three operands).
__device__ __forceinline__ float fmin_nan(float a, float b) {
  float d;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

__device__ __forceinline__ float fmin3_nan(float a, float b, float c) {
  float d;
  asm("min.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// -------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xFFFFFFFFu, x, o));
  return x;
}

__device__ __forceinline__ int warp_or(int x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x |= __shfl_xor_sync(0xFFFFFFFFu, x, o);
  return x;
}

__device__ __forceinline__ int warp_sum_i(int x) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
  return x;
}

__device__ __forceinline__ bool finite(float x) { return isfinite(x); }

}  // namespace ql
