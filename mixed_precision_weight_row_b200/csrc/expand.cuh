// Code expansion for the tensor-core decode kernels: one 32-code group of a
// packed row (B words) -> exact bf16 values in MMA fragment order.
//
// DynaQuant, "Custom kernel architecture": packed N-bit weights are expanded
// in registers to a tensor-core format.  The schemes (all exact):
//   * b = 4: the nibbles of codes k and k+4 sit 16 bits apart in a packed
//     word, so one shift and one LOP3 give two bf16 values 128 + u'
//     (u' = offset-binary code, OR-ed into the mantissa of 128.0);
//   * b = 8: likewise for the low and the high nibbles of bytes k and k+2;
//     q = 16*hi + lo, both parts fed to the same accumulator;
//   * b = 5..7: codes k and k+1 are brought to bits 0 and 16 with one funnel
//     shift, one shift and two LOP3s;
//   * b >= 9: the offset-binary code is split into 7-bit fields (weights 1,
//     128, 16384), each exact in bf16, one MMA per field.
// A bf16x2 FMA on the FMA pipe removes the 128 offset and applies the field
// weight, so every A operand is the exact code value.  The order of k inside
// a 16-wide MMA step is free; x fragments are permuted to match.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include <utility>

namespace mpw {
namespace dec {

enum Scheme { kNib4, kNib8, kAdj1, kAdjSplit };

template <int B>
struct Exp {
  static constexpr Scheme scheme = B == 4 ? kNib4 : (B == 8 ? kNib8 : (B <= 7 ? kAdj1 : kAdjSplit));
  static constexpr int parts = B == 4 ? 1 : (B == 8 ? 2 : (B <= 7 ? 1 : (B <= 14 ? 2 : 3)));
};

__device__ __forceinline__ uint32_t bf2_fma(uint32_t a, uint32_t mul, uint32_t add) {
  __nv_bfloat162 r = __hfma2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                             *reinterpret_cast<const __nv_bfloat162*>(&mul),
                             *reinterpret_cast<const __nv_bfloat162*>(&add));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// bf16 bit patterns used below (exact values)
constexpr uint32_t bf16_bits_of(int v) {
  // v is an integer with at most 8 significant bits and |v| < 2^24 (exact in bf16)
  if (v == 0) return 0u;
  uint32_t s = v < 0 ? 0x8000u : 0u;
  uint32_t a = static_cast<uint32_t>(v < 0 ? -v : v);
  int e = 0;
  while ((a >> e) > 1) ++e;                 // 2^e <= a < 2^(e+1)
  uint32_t mant = e >= 7 ? (a >> (e - 7)) & 0x7Fu : (a << (7 - e)) & 0x7Fu;
  return s | (static_cast<uint32_t>(127 + e) << 7) | mant;
}
constexpr uint32_t pair_of(int v) { return bf16_bits_of(v) | (bf16_bits_of(v) << 16); }

// Pair of fields of codes c and c+1 (adjacent in the stream) starting at bit
// offset f0 within each code, nb bits wide, as bf16 values 128 + field (with
// the bits of `flip` XOR-ed into each field).  t holds code c at bit 0 and
// code c+1 at bit B.
// One LOP3: (a & b) ^ c.
__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// Low half from a, high half from b (one PRMT).
__device__ __forceinline__ uint32_t merge_halves(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, 0x7610;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

template <int B, int F0, int NB, uint32_t FLIP>
__device__ __forceinline__ uint32_t adj_pair(uint32_t t) {
  const uint32_t a = F0 == 0 ? t : (t >> F0);
  constexpr int sh = 16 - B - F0;  // where code c+1's field must move to reach bit 16
  // a left shift is a multiply, which the FMA pipe can take off the ALU pipe
  const uint32_t b = sh >= 0 ? (t * (1u << (sh >= 0 ? sh : 0))) : (t >> (sh < 0 ? -sh : 0));
  constexpr uint32_t fm = ((1u << NB) - 1u) | (((1u << NB) - 1u) << 16);
  constexpr uint32_t xm = 0x43004300u | FLIP | (FLIP << 16);
  return and_xor(merge_halves(a, b), fm, xm);
}

// t = bits [o, o+32) of the group's words (code-aligned window)
template <int B>
__device__ __forceinline__ uint32_t window(const uint32_t (&w)[B + 1], int o) {
  const int i = o >> 5, r = o & 31;
  return r == 0 ? w[i] : __funnelshift_r(w[i], w[i + 1], r);
}

// Expands one 32-code group (B words) into parts x 16 bf16x2 registers; pair
// p feeds MMA step p/2 (low / high k half).  All values are exact integers.
template <int B>
__device__ __forceinline__ void expand_group(const uint32_t (&w)[B + 1], uint32_t (&v)[Exp<B>::parts][16]) {
  constexpr Scheme S = Exp<B>::scheme;
  if constexpr (S == kNib4) {
    // word i: codes 8i..8i+7; pair p = 4i+j = (code 8i+j, code 8i+j+4)
    const uint32_t off = pair_of(-136);  // -(128 + 8)
    const uint32_t one = pair_of(1);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t r = ((w[i] >> (4 * j)) & 0x000F000Fu) ^ 0x43084308u;
        v[0][4 * i + j] = bf2_fma(r, one, off);
      }
  } else if constexpr (S == kNib8) {
    // word i: codes 4i..4i+3 (bytes); pair p = 2i+j = (code 4i+j, code 4i+j+2)
    // q = 16*hi + lo with lo = low nibble (0..15), hi = high nibble (signed)
    const uint32_t one = pair_of(1), m128 = pair_of(-128);
    const uint32_t sixteen = pair_of(16), m2176 = pair_of(-2176);
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint32_t lo = ((w[i] >> (8 * j)) & 0x000F000Fu) | 0x43004300u;
        const uint32_t hi = ((w[i] >> (8 * j + 4)) & 0x000F000Fu) ^ 0x43084308u;
        v[0][2 * i + j] = bf2_fma(lo, one, m128);        // lo
        v[1][2 * i + j] = bf2_fma(hi, sixteen, m2176);   // 16 * hi
      }
  } else if constexpr (S == kAdj1) {
    constexpr int Q1 = 1 << (B - 1);
    const uint32_t one = pair_of(1), off = pair_of(-(128 + Q1));
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      const uint32_t t = window<B>(w, 2 * p * B);
      v[0][p] = bf2_fma(adj_pair<B, 0, B, (1u << (B - 1))>(t), one, off);
    }
  } else {
    // offset-binary u' = u ^ 2^(B-1) split into 7-bit fields
    const uint32_t one = pair_of(1), m128 = pair_of(-128);
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      const uint32_t t = window<B>(w, 2 * p * B);
      v[0][p] = bf2_fma(adj_pair<B, 0, 7, 0u>(t), one, m128);  // lo7
      if constexpr (B <= 14) {
        // 128 * (mid - 2^(B-8)); the sign flip of u' lands in this field
        constexpr int NB = B - 7;
        v[1][p] = bf2_fma(adj_pair<B, 7, NB, (1u << (NB - 1))>(t), pair_of(128),
                          pair_of(-128 * (128 + (1 << (B - 8)))));
      } else {
        v[1][p] = bf2_fma(adj_pair<B, 7, 7, 0u>(t), pair_of(128), pair_of(-128 * 128));
        // top bit (with the flip): 16384 * (top - 1)
        v[2][p] = bf2_fma(adj_pair<B, 14, 1, 1u>(t), pair_of(16384), pair_of(-16384 * 129));
      }
    }
  }
}

// Permutes the raw x pairs (x[2m], x[2m+1]) of a group into the k order of
// the expansion scheme.
template <int B>
__device__ __forceinline__ void permute_x(uint32_t (&xw)[16]) {
  constexpr Scheme S = Exp<B>::scheme;
  if constexpr (S == kNib4) {
    uint32_t o[16];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        o[4 * i + j] = __byte_perm(xw[4 * i + (j >> 1)], xw[4 * i + 2 + (j >> 1)], (j & 1) ? 0x7632 : 0x5410);
#pragma unroll
    for (int p = 0; p < 16; ++p) xw[p] = o[p];
  } else if constexpr (S == kNib8) {
    uint32_t o[16];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j) o[2 * i + j] = __byte_perm(xw[2 * i], xw[2 * i + 1], j ? 0x7632 : 0x5410);
#pragma unroll
    for (int p = 0; p < 16; ++p) xw[p] = o[p];
  }
}

// ---------------------------------------------------------------------------
// Paired-halves layout (a re-ordering of the canonical bits, K % 32 == 0):
// word h of a group holds half-word h of the stream of its even codes in the
// low 16 bits and half-word h of the stream of its odd codes in the high 16
// bits; code i of a stream occupies bits [i*B, i*B+B) of that stream.  The
// two codes of pair i = (2i, 2i+1) therefore sit at the same offset in the
// two halves of one word -- or, when the field crosses a half-word boundary,
// of two consecutive words -- so a shift and one LOP3 (two of each when the
// field crosses) give their bf16x2 pair, already in the k order of the raw x
// pairs (x[2i], x[2i+1]): no x permutation.
// ---------------------------------------------------------------------------

// Field [F0, F0+NB) of both codes of pair I as bf16 values 128 + field, the
// top bit of the field flipped when SIGNED (two's complement -> offset binary).
template <int B, int I, int F0, int NB, bool SIGNED>
__device__ __forceinline__ uint32_t paired_field(const uint32_t (&w)[B + 1]) {
  constexpr int o = I * B + F0;
  constexpr int h = o >> 4, r = o & 15;
  constexpr uint32_t fm = ((1u << NB) - 1u) * 0x10001u;
  constexpr uint32_t xm = 0x43004300u | (SIGNED ? (1u << (NB - 1)) * 0x10001u : 0u);
  uint32_t t;
  if constexpr (r + NB <= 16) {
    t = r == 0 ? w[h] : (w[h] >> r);
  } else if constexpr (r >= 8 && r + NB <= 24) {
    // the field lies in the top byte of each half of word h and the bottom
    // byte of each half of word h+1: one byte permute gathers both halves'
    // 16-bit windows (even stream low, odd stream high), then one shift
    uint32_t u;
    asm("prmt.b32 %0, %1, %2, 0x6341;" : "=r"(u) : "r"(w[h]), "r"(w[h + 1]));
    t = u >> (r - 8);
  } else {
    // low part from word h, high part from word h+1, in both halves at once
    constexpr uint32_t sel = ((1u << (16 - r)) - 1u) * 0x10001u;
    t = ((w[h] >> r) & sel) | ((w[h + 1] << (16 - r)) & ~sel);
  }
  return and_xor(t, fm, xm);
}

template <int B, int I>
__device__ __forceinline__ void paired_pair(const uint32_t (&w)[B + 1], uint32_t (&v)[Exp<B>::parts][16]) {
  const uint32_t one = pair_of(1);
  if constexpr (B <= 7) {
    v[0][I] = bf2_fma(paired_field<B, I, 0, B, true>(w), one, pair_of(-(128 + (1 << (B - 1)))));
  } else if constexpr (B == 8) {
    // q = lo + 16 * hi: low nibble unsigned, high nibble signed
    v[0][I] = bf2_fma(paired_field<B, I, 0, 4, false>(w), one, pair_of(-128));
    v[1][I] = bf2_fma(paired_field<B, I, 4, 4, true>(w), pair_of(16), pair_of(-16 * 136));
  } else if constexpr (B <= 14) {
    // q = lo7 + 128 * hi with hi = the signed top B-7 bits
    v[0][I] = bf2_fma(paired_field<B, I, 0, 7, false>(w), one, pair_of(-128));
    v[1][I] = bf2_fma(paired_field<B, I, 7, B - 7, true>(w), pair_of(128),
                      pair_of(-128 * (128 + (1 << (B - 8)))));
  } else {
    // q = lo7 + 128 * mid7 + 16384 * (top' - 1), top' = flipped sign bit
    v[0][I] = bf2_fma(paired_field<B, I, 0, 7, false>(w), one, pair_of(-128));
    v[1][I] = bf2_fma(paired_field<B, I, 7, 7, false>(w), pair_of(128), pair_of(-128 * 128));
    v[2][I] = bf2_fma(paired_field<B, I, 14, 1, true>(w), pair_of(16384), pair_of(-16384 * 129));
  }
}

template <int B, int... I>
__device__ __forceinline__ void paired_all(const uint32_t (&w)[B + 1], uint32_t (&v)[Exp<B>::parts][16],
                                           std::integer_sequence<int, I...>) {
  (paired_pair<B, I>(w, v), ...);
}

// Expands one 32-code group of a paired-halves row; v[part][i] holds pair i
// = (code 2i, code 2i+1), the k order of the raw x pairs.
template <int B>
__device__ __forceinline__ void expand_paired(const uint32_t (&w)[B + 1], uint32_t (&v)[Exp<B>::parts][16]) {
  paired_all<B>(w, v, std::make_integer_sequence<int, 16>{});
}

// ---------------------------------------------------------------------------
// Adjacent-pair expansion for the prefill GEMM, whose A operand in tensor
// memory holds codes (2i, 2i+1) of a group in one 32-bit column.  A code is
// fed whole when it is exact in bf16 (b <= 9) and as lo7 + 128*hi otherwise
// (two MMAs into one accumulator); b = 8, 9 and the high part of b = 15 are
// assembled from two magic fields with a second bf16x2 FMA.
// ---------------------------------------------------------------------------

template <int B>
struct GemmParts {
  static constexpr int parts = B <= 9 ? 1 : 2;
};

// Field [F0, F0+NB) of codes 2I and 2I+1 as bf16 values 128 + field, for
// either layout.
template <int B, bool PAIRED, int I, int F0, int NB, bool SIGNED>
__device__ __forceinline__ uint32_t field2(const uint32_t (&w)[B + 1]) {
  if constexpr (PAIRED) {
    return paired_field<B, I, F0, NB, SIGNED>(w);
  } else {
    return adj_pair<B, F0, NB, (SIGNED ? (1u << (NB - 1)) : 0u)>(window<B>(w, 2 * I * B));
  }
}

template <int B, bool PAIRED, int I>
__device__ __forceinline__ void gemm_pair(const uint32_t (&w)[B + 1], uint32_t (&v)[GemmParts<B>::parts][16]) {
  const uint32_t one = pair_of(1);
  if constexpr (B <= 7) {
    v[0][I] = bf2_fma(field2<B, PAIRED, I, 0, B, true>(w), one, pair_of(-(128 + (1 << (B - 1)))));
  } else if constexpr (B <= 9) {
    // q = lo7 + 128 * hi fits bf16: t = 128 * hi - 128, then (128 + lo7) + t
    const uint32_t t = bf2_fma(field2<B, PAIRED, I, 7, B - 7, true>(w), pair_of(128),
                               pair_of(-128 * (129 + (1 << (B - 8)))));
    v[0][I] = bf2_fma(field2<B, PAIRED, I, 0, 7, false>(w), one, t);
  } else if constexpr (B <= 14) {
    v[0][I] = bf2_fma(field2<B, PAIRED, I, 0, 7, false>(w), one, pair_of(-128));
    v[1][I] = bf2_fma(field2<B, PAIRED, I, 7, B - 7, true>(w), pair_of(128),
                      pair_of(-128 * (128 + (1 << (B - 8)))));
  } else {
    // 128 * hi with hi = mid7 + 128 * (top' - 1): t = 16384 * top' - 32768,
    // then 128 * (128 + mid7) + t
    v[0][I] = bf2_fma(field2<B, PAIRED, I, 0, 7, false>(w), one, pair_of(-128));
    const uint32_t t = bf2_fma(field2<B, PAIRED, I, 14, 1, true>(w), pair_of(16384),
                               pair_of(-16384 * 128 - 32768));
    v[1][I] = bf2_fma(field2<B, PAIRED, I, 7, 7, false>(w), pair_of(128), t);
  }
}

template <int B, bool PAIRED, int... I>
__device__ __forceinline__ void gemm_all(const uint32_t (&w)[B + 1], uint32_t (&v)[GemmParts<B>::parts][16],
                                         std::integer_sequence<int, I...>) {
  (gemm_pair<B, PAIRED, I>(w, v), ...);
}

// One 32-code group -> 16 adjacent bf16x2 pairs per part (exact values).
template <int B, bool PAIRED>
__device__ __forceinline__ void gemm_expand_group(const uint32_t (&w)[B + 1],
                                                  uint32_t (&v)[GemmParts<B>::parts][16]) {
  gemm_all<B, PAIRED>(w, v, std::make_integer_sequence<int, 16>{});
}

// Bits of codes 2I and 2I+1 of a 32-code group at bit 0 of the low and of the
// high half of the result (the higher bits of each half are the neighbours'),
// for either layout.
template <int B, bool PAIRED, int I>
__device__ __forceinline__ uint32_t pair_window(const uint32_t (&w)[B + 1]) {
  if constexpr (PAIRED) {
    constexpr int o = I * B;
    constexpr int h = o >> 4, r = o & 15;
    if constexpr (r + B <= 16) {
      return r == 0 ? w[h] : (w[h] >> r);
    } else {
      constexpr uint32_t sel = ((1u << (16 - r)) - 1u) * 0x10001u;
      return ((w[h] >> r) & sel) | ((w[h + 1] << (16 - r)) & ~sel);
    }
  } else {
    const uint32_t t = window<B>(w, 2 * I * B);   // code 2I at bit 0, code 2I+1 at bit B
    return merge_halves(t, t << (16 - B));
  }
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

}  // namespace dec
}  // namespace mpw
