// Exact mean of bf16 values, rounded once to float32.
//
// "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破", section 三(一) item 1:
// K is smoothed by subtracting its per-channel mean over the tokens.  The mean
// is taken here as the exact sum of the N bf16 values divided by N, rounded to
// the nearest float32 (ties to even), so that it does not depend on the order
// of the additions.
//
// A finite bf16 value is (-1)^s * m * 2^(e - 134) with the 8-bit significand m
// (m < 256) and e = max(exponent field, 1).  In units of 2^-133 it is the
// integer m << (e - 1), at most 255 * 2^253; N < 2^31 of them sum to less than
// 2^292.  The sums are kept as two 320-bit magnitudes (positive and negative
// parts, five 64-bit limbs each, least significant first) and combined at the
// end.  Used by k_channel_mean for the channels whose float64 block sums cannot
// be shown to be exact; plain integer arithmetic, host and device.
#pragma once
#include <cstdint>
#include <cstring>

namespace sla {

constexpr int kWideLimbs = 5;

struct Wide320 {
  uint64_t w[kWideLimbs];
};

__host__ __device__ __forceinline__ void wide_zero(Wide320& a) {
#pragma unroll
  for (int i = 0; i < kWideLimbs; ++i) a.w[i] = 0;
}

// a += b
__host__ __device__ __forceinline__ void wide_add(Wide320& a, const Wide320& b) {
  uint64_t carry = 0;
#pragma unroll
  for (int i = 0; i < kWideLimbs; ++i) {
    const uint64_t s = a.w[i] + b.w[i];
    const uint64_t c1 = s < b.w[i] ? 1u : 0u;
    const uint64_t s2 = s + carry;
    const uint64_t c2 = s2 < carry ? 1u : 0u;
    a.w[i] = s2;
    carry = c1 | c2;
  }
}

// a += mag * 2^shift, mag < 2^8, 0 <= shift <= 253 (branch-free over the limbs)
__host__ __device__ __forceinline__ void wide_add_shifted(Wide320& a, uint64_t mag, int shift) {
  const int L = shift >> 6, off = shift & 63;
  const uint64_t lo = mag << off;
  const uint64_t hi = off != 0 ? (mag >> (64 - off)) : 0u;
  uint64_t carry = 0;
#pragma unroll
  for (int i = 0; i < kWideLimbs; ++i) {
    const uint64_t add = (i == L) ? lo : ((i == L + 1) ? hi : 0u);
    const uint64_t s = a.w[i] + add;
    const uint64_t c1 = s < add ? 1u : 0u;
    const uint64_t s2 = s + carry;
    const uint64_t c2 = s2 < carry ? 1u : 0u;
    a.w[i] = s2;
    carry = c1 | c2;
  }
}

// Adds one bf16 value (raw bits, finite) to the positive or the negative part.
__host__ __device__ __forceinline__ void wide_add_bf16(Wide320& pos, Wide320& neg, uint16_t bits) {
  const uint32_t ef = (bits >> 7) & 0xFFu;
  const uint32_t frac = bits & 0x7Fu;
  const uint64_t mag = ef != 0 ? (frac | 0x80u) : frac;
  const int shift = (ef != 0 ? int(ef) : 1) - 1;
  if (bits & 0x8000u)
    wide_add_shifted(neg, mag, shift);
  else
    wide_add_shifted(pos, mag, shift);
}

// a >= b
__host__ __device__ __forceinline__ bool wide_ge(const Wide320& a, const Wide320& b) {
  for (int i = kWideLimbs - 1; i >= 0; --i)
    if (a.w[i] != b.w[i]) return a.w[i] > b.w[i];
  return true;
}

// a - b for a >= b
__host__ __device__ __forceinline__ Wide320 wide_sub(const Wide320& a, const Wide320& b) {
  Wide320 r;
  uint64_t borrow = 0;
#pragma unroll
  for (int i = 0; i < kWideLimbs; ++i) {
    const uint64_t d = a.w[i] - b.w[i];
    const uint64_t b1 = a.w[i] < b.w[i] ? 1u : 0u;
    const uint64_t d2 = d - borrow;
    const uint64_t b2 = d < borrow ? 1u : 0u;
    r.w[i] = d2;
    borrow = b1 | b2;
  }
  return r;
}

// The float32 nearest to (pos - neg) * 2^-133 / n, ties to even (n >= 1).
//
// With M = |pos - neg|, the quotient Q = floor(M * 2^64 / n) and remainder R
// are formed by long division over 32-bit digits; for M >= 1, Q >= 2^33, so Q
// carries more than the 24 bits a float32 keeps (M * 2^64 < 2^356 fits in
// twelve digits).  The value is (Q + R/n) * 2^-197: the kept bits are those of
// Q from position `shift` = max(top bit - 23, 48) up (48 = the position of
// 2^-149, the float32 subnormal spacing); it rounds up when the first dropped
// bit is set and either a lower dropped bit, R, or the lowest kept bit is set.
__host__ __device__ inline float wide_mean_to_f32(const Wide320& pos, const Wide320& neg, uint32_t n) {
  const bool negative = !wide_ge(pos, neg);
  const Wide320 m = negative ? wide_sub(neg, pos) : wide_sub(pos, neg);
  uint32_t dig[12];   // M * 2^64, 32-bit digits, least significant first
  dig[0] = dig[1] = 0u;
#pragma unroll
  for (int i = 0; i < kWideLimbs; ++i) {
    dig[2 + 2 * i] = uint32_t(m.w[i]);
    dig[3 + 2 * i] = uint32_t(m.w[i] >> 32);
  }
  uint32_t q[12];
  uint64_t rem = 0;
  for (int i = 11; i >= 0; --i) {
    const uint64_t cur = (rem << 32) | dig[i];
    q[i] = uint32_t(cur / n);
    rem = cur % n;
  }
  int top = -1;
  for (int i = 11; i >= 0 && top < 0; --i)
    if (q[i] != 0u) {
      int b = 31;
      while (((q[i] >> b) & 1u) == 0u) --b;
      top = 32 * i + b;
    }
  const uint32_t sign = negative ? 0x80000000u : 0u;
  if (top < 0) return 0.0f;   // M == 0
  auto bit = [&](int p) -> uint32_t { return (q[p >> 5] >> (p & 31)) & 1u; };
  int shift = top - 23 > 48 ? top - 23 : 48;
  uint32_t mant = 0u;
  for (int p = top; p >= shift; --p) mant = (mant << 1) | bit(p);
  const uint32_t half = bit(shift - 1);
  bool lower = rem != 0;
  for (int p = shift - 2; p >= 0 && !lower; --p) lower = bit(p) != 0u;
  if (half && (lower || (mant & 1u))) ++mant;
  if (mant == (1u << 24)) {
    mant = 1u << 23;
    ++shift;
  }
  uint32_t bits;
  if (mant >= (1u << 23))
    bits = sign | (uint32_t(shift - 47) << 23) | (mant - (1u << 23));
  else
    bits = sign | mant;   // subnormal (shift == 48) or zero
  float f;
  memcpy(&f, &bits, 4);
  return f;
}

}  // namespace sla
