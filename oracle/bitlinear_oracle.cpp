// BitLinear forward oracle: plain, slow, single-threaded C++17 restatement of what
// BitNet b1.58 ("The Era of 1-bit LLMs: All Large Language Models are in 1.58 Bits")
// computes in one BitLinear layer.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the library path may link, load or call this
// file; only the tests, the smoke check and the benchmark's CPU-baseline leg do.
// It shares no code, header, table or helper with the CUDA library.
//
// Sources (page, section), restated:
//  - every weight of the model takes one of the three values -1, 0, +1:
//    searcharxiv.com abstract page, Abstract.
//  - BitLinear takes the place of nn.Linear; an absmean quantization function limits
//    the weights to {-1, 0, +1} and the activations are held in 8 bits: dmarx anthology
//    record LIT-380, Key takeaways, bullet 1.
//  - with ternary weights the matrix product needs only integer additions (and
//    subtractions), no multiplications: LIT-380, Key takeaways, bullet 4.
//  - a 1.58-bit weight is stored in 2 bits in practice: hackerpaper HN page, thread 17.
// The pages print no formula. The formulas below are the plainest reading of
// absmean weights and 8-bit activations: gamma = mean|W|, W~ = RoundClip(W/(gamma+eps), -1, 1),
// per-token absmax int8 in [-127, 127], int32 accumulation, rescale by gamma*absmax/127,
// round-half-to-even everywhere. Every arithmetic step is fp32 IEEE round-to-nearest-even
// with no contraction (build with -ffp-contract=off, no fast-math).
//
// Packed weight format (the library's 2-bit storage of each trit):
//  - each trit c in {-1,0,+1} is stored as the 2-bit unsigned code u = c + 1 (0,1,2; 3 is
//    never written);
//  - row n of W[N][K] occupies K/4 bytes starting at byte n*K/4 (K a multiple of 16);
//  - the little-endian 32-bit word g of a row holds trits k = 16g .. 16g+15, trit
//    k = 16g + 4j + i (i, j in 0..3) sitting in bits 8i+2j and 8i+2j+1 of that word,
//    i.e. in byte 4g+i of the row at bit 2j.
//
// Parity pins for every function live in tests/test_oracle.py.

#include <cstdint>
#include <cstring>
#include <cfenv>
#include <cmath>
#include <vector>

namespace {

// Widen element i of a buffer holding fp32 (dtype 0) or bf16 (dtype 1) values to fp32.
// bf16 -> fp32 is exact: the bf16 bits are the top 16 bits of the fp32 pattern.
float load_value(const void* p, int dtype, int64_t i) {
  if (dtype == 0) return static_cast<const float*>(p)[i];
  uint32_t bits = static_cast<uint32_t>(static_cast<const uint16_t*>(p)[i]) << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return f;
}

uint32_t float_bits(float f) {
  uint32_t b;
  std::memcpy(&b, &f, sizeof b);
  return b;
}

// Round half to even: the C library's nearbyint under the default rounding mode
// (FE_TONEAREST, checked by every entry point that uses it). q is finite.
float round_half_even(float q) { return std::nearbyint(q); }

bool rounding_mode_is_nearest() { return std::fegetround() == FE_TONEAREST; }

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------------------
// Step W1+W2: gamma = mean |W| over the whole matrix (absmean, LIT-380 bullet 1).
//
// The pages give no summation order, so the sum of |w| is formed EXACTLY and rounded
// once: every |w| = m * 2^(max(e,1) - 150) with biased exponent e and integer mantissa
// m < 2^24. Bucket B[e] accumulates the integer mantissas of exponent e (uint64 is enough
// for n <= 2^31). The exact sum S * 2^149 = sum_e B[e] * 2^(max(e,1) - 1) is built in a
// multi-word integer, rounded once to double (round half to even), divided by n in double
// and rounded to float. The two halves are separate functions so that the buckets of the
// parts of a matrix split over several devices can be added (integers) before gamma is
// formed once for the whole matrix.

// First half: the 256 exponent buckets of the n values (bucket[0] stays 0; subnormals go
// to bucket[1]). Returns 0, or 1 if any |w| is Inf or NaN.
int oracle_abs_buckets(const void* W, int dtype, int64_t n, uint64_t* bucket) {
  for (int e = 0; e < 256; ++e) bucket[e] = 0;
  for (int64_t i = 0; i < n; ++i) {
    uint32_t bits = float_bits(load_value(W, dtype, i)) & 0x7fffffffu;
    uint32_t e = bits >> 23;
    if (e == 255u) return 1;
    uint32_t m = bits & 0x7fffffu;
    if (e != 0u) m |= 0x800000u;
    bucket[e == 0u ? 1u : e] += m;  // subnormals share the unit 2^-149 with e = 1
  }
  return 0;
}

// Second half: gamma from the buckets of n values in all.
void oracle_absmean_from_buckets(const uint64_t* bucket, int64_t n, float* gamma_out) {

  // Exact integer S * 2^149 as little-endian 32-bit words (512 bits is plenty:
  // the largest term is < 2^55 * 2^253).
  const int kWords = 16;
  uint32_t big[kWords];
  for (int w = 0; w < kWords; ++w) big[w] = 0;
  for (int e = 1; e < 255; ++e) {
    if (bucket[e] == 0) continue;
    int shift = e - 1;
    int word = shift / 32;
    int bit = shift % 32;
    // the term bucket[e] << bit spans at most three 32-bit words
    uint64_t lo = bucket[e] << bit;                                // low 64 bits
    uint64_t hi = (bit == 0) ? 0 : (bucket[e] >> (64 - bit));      // the rest (< 2^32)
    uint32_t parts[3] = {static_cast<uint32_t>(lo), static_cast<uint32_t>(lo >> 32),
                         static_cast<uint32_t>(hi)};
    uint64_t carry = 0;
    for (int p = 0; word + p < kWords; ++p) {
      uint64_t add = (p < 3) ? parts[p] : 0;
      if (p >= 3 && carry == 0) break;
      uint64_t s = static_cast<uint64_t>(big[word + p]) + add + carry;
      big[word + p] = static_cast<uint32_t>(s);
      carry = s >> 32;
    }
  }

  // Highest set bit of the big integer.
  int top = -1;
  for (int w = kWords - 1; w >= 0 && top < 0; --w) {
    if (big[w] != 0) {
      for (int b = 31; b >= 0; --b) {
        if ((big[w] >> b) & 1u) { top = 32 * w + b; break; }
      }
    }
  }
  double sum;
  if (top < 0) {
    sum = 0.0;
  } else {
    auto bit_at = [&](int pos) -> uint64_t {
      return (pos < 0) ? 0u : ((big[pos / 32] >> (pos % 32)) & 1u);
    };
    // 53-bit significand = bits top .. top-52 (missing low positions read as 0)
    uint64_t mant = 0;
    for (int pos = top; pos >= top - 52; --pos) mant = (mant << 1) | bit_at(pos);
    int low = top - 52;  // weight of the significand's last bit is 2^low
    if (low > 0) {
      uint64_t half = bit_at(low - 1);
      uint64_t sticky = 0;
      for (int pos = low - 2; pos >= 0; --pos) sticky |= bit_at(pos);
      if (half && (sticky || (mant & 1u))) mant += 1;  // ties to even
    }
    // value = mant * 2^low * 2^-149; mant <= 2^53, so this product is exact
    sum = std::ldexp(static_cast<double>(mant), low - 149);
  }
  double mean = sum / static_cast<double>(n);
  *gamma_out = static_cast<float>(mean);
}

// gamma = mean |W| over the n values: both halves. Returns 0, or 1 for Inf/NaN.
int oracle_absmean(const void* W, int dtype, int64_t n, float* gamma_out) {
  uint64_t bucket[256];
  if (oracle_abs_buckets(W, dtype, n, bucket) != 0) return 1;
  oracle_absmean_from_buckets(bucket, n, gamma_out);
  return 0;
}

// Steps W3+W4: ternary code c = RoundClip(w / (gamma + eps), -1, 1).
// d = gamma + eps in fp32; w / d is the correctly rounded fp32 quotient; rounding is
// half-to-even; the result is clipped to [-1, 1]. If d == 0 (gamma = 0 and eps = 0)
// every code is 0. Non-finite w is not supported by the method (callers check absmean).
// Returns 0, or 3 if the FPU rounding mode is not round-to-nearest.
int oracle_ternarize(const void* W, int dtype, int64_t n, float gamma, float eps,
                     int8_t* codes) {
  if (!rounding_mode_is_nearest()) return 3;
  float d = gamma + eps;
  for (int64_t i = 0; i < n; ++i) {
    if (d == 0.0f) { codes[i] = 0; continue; }
    float w = load_value(W, dtype, i);
    float q = w / d;
    int c;
    if (q >= 1.5f) {
      c = 1;  // RoundClip saturates; also covers q = +inf
    } else if (q <= -1.5f) {
      c = -1;
    } else {
      float r = round_half_even(q);
      c = static_cast<int>(r);
      if (c > 1) c = 1;
      if (c < -1) c = -1;
    }
    codes[i] = static_cast<int8_t>(c);
  }
  return 0;
}

// Step W5: 2-bit packing of codes[N][K] (layout in the file header). K % 16 == 0.
void oracle_pack(const int8_t* codes, int64_t N, int64_t K, uint8_t* packed) {
  const int64_t row_bytes = K / 4;
  for (int64_t b = 0; b < N * row_bytes; ++b) packed[b] = 0;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      uint32_t u = static_cast<uint32_t>(codes[n * K + k] + 1);
      int64_t g = k / 16;
      int64_t j = (k % 16) / 4;
      int64_t i = k % 4;
      packed[n * row_bytes + 4 * g + i] |= static_cast<uint8_t>(u << (2 * j));
    }
  }
}

// Inverse of oracle_pack. Returns 0, or 1 if a 2-bit field holds the unused code 3.
int oracle_unpack(const uint8_t* packed, int64_t N, int64_t K, int8_t* codes) {
  const int64_t row_bytes = K / 4;
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      int64_t g = k / 16;
      int64_t j = (k % 16) / 4;
      int64_t i = k % 4;
      uint32_t u = (packed[n * row_bytes + 4 * g + i] >> (2 * j)) & 3u;
      if (u == 3u) return 1;
      codes[n * K + k] = static_cast<int8_t>(static_cast<int>(u) - 1);
    }
  }
  return 0;
}

// ---------------------------------------------------------------------------------------
// Base-3 packing, 5 trits per byte (hackerpaper HN page, thread 3: 3^5 = 243 <= 256, so
// five ternary digits fit a byte, 1.6 bits per weight instead of 2).
//
// Layout (the library's base-3 format): row n of W[N][K] occupies R = ceil(K / 80) * 16
// bytes at byte offset n * R, in 16-byte chunks of 80 trits. Byte i (0..15) of chunk j
// holds the five trits k = 80 j + 16 p + i, p = 0..4 (trits past K are 0). With
// u_p = c_p + 1 in {0, 1, 2}, the byte stores the base-3 number v = sum_p u_p 3^(4 - p)
// (u_0 the leading digit) as the fixed-point value B = ceil(256 v / 243), in 0..255.
// Decoding: u_p = floor(B 3^(p+1) / 256) mod 3, exactly, for every v in 0..242.

// Bytes per row of the base-3 format.
int64_t oracle_base3_row_bytes(int64_t K) { return (K + 79) / 80 * 16; }

// codes [N][K] int8 in {-1,0,1} -> packed3 [N][R] (R = oracle_base3_row_bytes(K)).
void oracle_pack_base3(const int8_t* codes, int64_t N, int64_t K, uint8_t* packed3) {
  const int64_t R = oracle_base3_row_bytes(K);
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t j = 0; j < R / 16; ++j) {
      for (int i = 0; i < 16; ++i) {
        int64_t v = 0;
        for (int p = 0; p < 5; ++p) {
          const int64_t k = 80 * j + 16 * p + i;
          const int u = (k < K) ? codes[n * K + k] + 1 : 1;
          v = 3 * v + u;  // u_0 ends up as the leading digit
        }
        packed3[n * R + 16 * j + i] = static_cast<uint8_t>((256 * v + 242) / 243);
      }
    }
  }
}

// packed3 [N][R] -> codes [N][K]. Returns 0, or 1 if a decoded byte is not the encoding of
// any v (the byte is not ceil(256 v / 243) of its decoded v) or a trit past K is non-zero.
int oracle_unpack_base3(const uint8_t* packed3, int64_t N, int64_t K, int8_t* codes) {
  const int64_t R = oracle_base3_row_bytes(K);
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t j = 0; j < R / 16; ++j) {
      for (int i = 0; i < 16; ++i) {
        const int64_t B = packed3[n * R + 16 * j + i];
        int64_t v = 0;
        int64_t pow3 = 3;
        for (int p = 0; p < 5; ++p, pow3 *= 3) {
          const int u = static_cast<int>((B * pow3 / 256) % 3);
          v = 3 * v + u;
          const int64_t k = 80 * j + 16 * p + i;
          if (k < K) codes[n * K + k] = static_cast<int8_t>(u - 1);
          else if (u != 1) return 1;
        }
        if ((256 * v + 242) / 243 != B) return 1;
      }
    }
  }
  return 0;
}

// ---------------------------------------------------------------------------------------
// BitLinear backward for quantization-aware training with the straight-through estimator
// (hackerpaper HN page, thread 21: the rounding steps are passed straight through in the
// backward pass; LIT-380 bullet 1: the model is trained with these quantizers in place).
// The forward is y = X~ W~^T with the dequantized operands X~[t,k] = q[t,k] s_t and
// W~[n,k] = gamma c[n,k]; the estimator treats both quantizers as the identity, so for an
// upstream gradient G = dL/dy [M][N]:
//   dL/dx = G W~       -> grad_x[t,k] = gamma * sum_n G[t,n] c[n,k]
//   dL/dW = G^T X~     -> grad_w[n,k] = sum_t G[t,n] X~[t,k]
// G is bf16 (dtype 1) or fp32 (dtype 0). X~ is taken as the library holds it, in bf16:
// X~[t,k] = bf16(fl32(q[t,k] * s_t)) (round half to even). Sums are formed in double
// (every product is exact there), the results are doubles.

// dequantized activations X~ [M][K] as bf16 bit patterns
void oracle_dequant_acts_bf16(const int8_t* q, const float* scale, int64_t M, int64_t K,
                              uint16_t* out) {
  for (int64_t t = 0; t < M; ++t) {
    for (int64_t k = 0; k < K; ++k) {
      const float v = static_cast<float>(q[t * K + k]) * scale[t];
      uint32_t b = float_bits(v);
      uint32_t lower = b & 0xffffu, upper = b >> 16;
      if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1;
      out[t * K + k] = static_cast<uint16_t>(upper);
    }
  }
}

void oracle_ste_grad_x(const void* G, int dtype, const int8_t* codes, float gamma, int64_t M,
                       int64_t N, int64_t K, double* grad_x) {
  for (int64_t t = 0; t < M; ++t) {
    for (int64_t k = 0; k < K; ++k) {
      double s = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        const int8_t c = codes[n * K + k];
        if (c == 1) s += static_cast<double>(load_value(G, dtype, t * N + n));
        else if (c == -1) s -= static_cast<double>(load_value(G, dtype, t * N + n));
      }
      grad_x[t * K + k] = static_cast<double>(gamma) * s;
    }
  }
}

void oracle_ste_grad_w(const void* G, int dtype, const uint16_t* xt_bf16, int64_t M, int64_t N,
                       int64_t K, double* grad_w) {
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      double s = 0.0;
      for (int64_t t = 0; t < M; ++t)
        s += static_cast<double>(load_value(G, dtype, t * N + n)) *
             static_cast<double>(load_value(xt_bf16, 1, t * K + k));
      grad_w[n * K + k] = s;
    }
  }
}

// Steps X1+X2: per-token absmax int8 quantization (8-bit activations, LIT-380
// bullet 1). a_t = max_k |x[t,k]|; r_t = 127 / a_t (fp32); q = clip(rne(x * r_t), -127, 127);
// s_t = a_t / 127 (fp32). A zero row gives q = 0 and s_t = 0; an exactly-zero element
// gives q = 0. Returns 0, 1 if x holds Inf or NaN, 3 if the rounding mode is not nearest.
//
// Split in two steps (X1, then X2 given a_t) so that a row held in K-shards on several
// devices can form a_t as the maximum of the shards' maxima first.

// X1 alone: amax[t] = max_k |x[t,k]|. Returns 0, or 1 if x holds Inf or NaN.
int oracle_act_absmax(const void* x, int dtype, int64_t M, int64_t K, float* amax) {
  for (int64_t t = 0; t < M; ++t) {
    float a = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float v = std::fabs(load_value(x, dtype, t * K + k));
      if (!(v <= 3.4028234663852886e38f)) return 1;  // Inf or NaN
      if (v > a) a = v;
    }
    amax[t] = a;
  }
  return 0;
}

// X2 with a_t given (a_t >= 0 and finite; values above a_t clip to +-127).
// Returns 0, or 3 if the rounding mode is not nearest.
int oracle_quantize_acts_absmax(const void* x, int dtype, int64_t M, int64_t K,
                                const float* amax, int8_t* q, float* scale) {
  if (!rounding_mode_is_nearest()) return 3;
  for (int64_t t = 0; t < M; ++t) {
    const float a = amax[t];
    if (a == 0.0f) {
      for (int64_t k = 0; k < K; ++k) q[t * K + k] = 0;
      scale[t] = 0.0f;
      continue;
    }
    float r = 127.0f / a;
    scale[t] = a / 127.0f;
    for (int64_t k = 0; k < K; ++k) {
      float v = load_value(x, dtype, t * K + k);
      int c;
      if (v == 0.0f) {
        c = 0;
      } else {
        float p = v * r;
        if (p >= 127.5f) {
          c = 127;
        } else if (p <= -127.5f) {
          c = -127;
        } else {
          c = static_cast<int>(round_half_even(p));
          if (c > 127) c = 127;
          if (c < -127) c = -127;
        }
      }
      q[t * K + k] = static_cast<int8_t>(c);
    }
  }
  return 0;
}

// X1 then X2 on whole rows. Returns 0, 1 if x holds Inf or NaN, 3 if the rounding mode is
// not nearest.
int oracle_quantize_acts(const void* x, int dtype, int64_t M, int64_t K, int8_t* q,
                         float* scale) {
  std::vector<float> amax(static_cast<size_t>(M));
  if (oracle_act_absmax(x, dtype, M, K, amax.data()) != 0) return 1;
  return oracle_quantize_acts_absmax(x, dtype, M, K, amax.data(), q, scale);
}

// Step C1: acc[t,n] = sum over k with c = +1 of q[t,k] minus sum over k with c = -1 of
// q[t,k]: additions and subtractions only, no multiplication (LIT-380 bullet 4). Zero codes
// are skipped, the feature filtering of LIT-380 bullet 2. codes is the unpacked [N][K] array.
void oracle_contract_i32(const int8_t* q, const int8_t* codes, int64_t M, int64_t N,
                         int64_t K, int32_t* acc) {
  for (int64_t t = 0; t < M; ++t) {
    for (int64_t n = 0; n < N; ++n) {
      int32_t s = 0;
      for (int64_t k = 0; k < K; ++k) {
        int8_t c = codes[n * K + k];
        if (c == 1) {
          s += q[t * K + k];
        } else if (c == -1) {
          s -= q[t * K + k];
        }
      }
      acc[t * N + n] = s;
    }
  }
}

// Step R1: y[t,n] = float(acc[t,n]) * (s_t * gamma), both products fp32 round-to-nearest.
void oracle_rescale(const int32_t* acc, const float* scale, float gamma, int64_t M,
                    int64_t N, float* y) {
  for (int64_t t = 0; t < M; ++t) {
    float f = scale[t] * gamma;
    for (int64_t n = 0; n < N; ++n) y[t * N + n] = static_cast<float>(acc[t * N + n]) * f;
  }
}

// fp32 -> bf16 with round half to even (bf16 outputs are the RNE of the fp32 result).
void oracle_to_bf16(const float* y, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) {
    uint32_t b = float_bits(y[i]);
    if ((b & 0x7fffffffu) > 0x7f800000u) {  // NaN stays NaN
      out[i] = static_cast<uint16_t>((b >> 16) | 0x40u);
      continue;
    }
    uint32_t lower = b & 0xffffu;
    uint32_t upper = b >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1;
    out[i] = static_cast<uint16_t>(upper);
  }
}

// Whole weight path: absmean, ternarize, pack. Returns 0, 1 (non-finite W) or 3.
int oracle_quantize_weights(const void* W, int dtype, int64_t N, int64_t K, float eps,
                            uint8_t* packed, float* gamma_out, int8_t* codes_scratch) {
  float gamma;
  if (oracle_absmean(W, dtype, N * K, &gamma) != 0) return 1;
  if (oracle_ternarize(W, dtype, N * K, gamma, eps, codes_scratch) != 0) return 3;
  oracle_pack(codes_scratch, N, K, packed);
  *gamma_out = gamma;
  return 0;
}

// Whole forward: quantize x, unpack W, contract, rescale. y is fp32 [M][N].
// codes_scratch holds N*K int8, q_scratch M*K int8, acc_scratch M*N int32,
// scale_scratch M floats. Returns 0, 1 (non-finite x), 2 (bad packed code) or 3
// (rounding mode not nearest).
int oracle_forward(const void* x, int dtype, const uint8_t* packed, float gamma, int64_t M,
                   int64_t N, int64_t K, float* y, int8_t* codes_scratch, int8_t* q_scratch,
                   int32_t* acc_scratch, float* scale_scratch) {
  int rc = oracle_quantize_acts(x, dtype, M, K, q_scratch, scale_scratch);
  if (rc != 0) return rc;
  if (oracle_unpack(packed, N, K, codes_scratch) != 0) return 2;
  oracle_contract_i32(q_scratch, codes_scratch, M, N, K, acc_scratch);
  oracle_rescale(acc_scratch, scale_scratch, gamma, M, N, y);
  return 0;
}

}  // extern "C"
