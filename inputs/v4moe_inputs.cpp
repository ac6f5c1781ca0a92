// Seeded synthetic inputs for the routed MoE layer of DeepSeek-V4-Flash.
//
// This file draws random numbers and encodes them into the storage formats the
// layer consumes (bf16 activations, MXFP4 expert weights, int8 per-channel
// shared-expert weights, Zipf token ids and a token-id -> expert hash table).
// It holds none of the layer's arithmetic: no decode table, no routing, no
// GEMM. Both the CPU oracle and the CUDA library consume its bytes.
//
// Random stream: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
// numbers: as easy as 1, 2, 3", SC'11), key = (seed, tensor tag), counter =
// (block index lo, block index hi, sub-stream, 0). Every output element is a
// pure function of (seed, tag, element index), so results do not depend on the
// number of threads used to produce them.
//
// Normal variates: Box-Muller on the four 32-bit lanes of one Philox block.
//
// Encodings (the recipe of the synthetic workloads):
//  * bf16: round-to-nearest-even of the fp32 draw.
//  * MXFP4 (OCP Microscaling v1.0 element type E2M1, E8M0 block scale, block
//    32 along K): shared exponent X = floor(log2(amax)) - 2, stored as
//    X + 127 clamped to [0, 254]; each element v/2^X rounds to the nearest
//    E2M1 magnitude, ties to the even code, saturating at 6. Codes are packed
//    two per byte, the element with the even K index in the low nibble.
//  * int8 per output channel, symmetric: scale = amax/127 in fp32,
//    q = clamp(rne(w/scale), -127, 127); a zero row gets scale 1.
//  * Zipf(s) token ids over ranks 1..V by inverse CDF (fp64 CDF, binary
//    search); id = rank - 1.
//  * tid2eid rows: k distinct experts from a partial Fisher-Yates shuffle of
//    0..E-1 driven by Philox draws.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

constexpr uint32_t kPhiloxM0 = 0xD2511F53u;
constexpr uint32_t kPhiloxM1 = 0xCD9E8D57u;
constexpr uint32_t kPhiloxW0 = 0x9E3779B9u;
constexpr uint32_t kPhiloxW1 = 0xBB67AE85u;

struct Block4 {
  uint32_t v[4];
};

inline Block4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0,
                            uint32_t k1) {
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = uint64_t(kPhiloxM0) * c0;
    const uint64_t p1 = uint64_t(kPhiloxM1) * c2;
    const uint32_t hi0 = uint32_t(p0 >> 32), lo0 = uint32_t(p0);
    const uint32_t hi1 = uint32_t(p1 >> 32), lo1 = uint32_t(p1);
    const uint32_t n0 = hi1 ^ c1 ^ k0;
    const uint32_t n1 = lo1;
    const uint32_t n2 = hi0 ^ c3 ^ k1;
    const uint32_t n3 = lo0;
    c0 = n0;
    c1 = n1;
    c2 = n2;
    c3 = n3;
    k0 += kPhiloxW0;
    k1 += kPhiloxW1;
  }
  return Block4{{c0, c1, c2, c3}};
}

struct Stream {
  uint32_t k0, k1;
  Stream(uint64_t seed, uint32_t tag) : k0(uint32_t(seed) ^ uint32_t(seed >> 32) * 0x9E3779B1u), k1(tag) {}
  Block4 block(uint64_t idx, uint32_t sub = 0) const {
    return philox4x32_10(uint32_t(idx), uint32_t(idx >> 32), sub, 0u, k0, k1);
  }
};

// Uniform in (0, 1) from the top 24 bits of a lane.
inline float u01(uint32_t a) { return (float(a >> 8) + 0.5f) * (1.0f / 16777216.0f); }

// Four standard normals from one Philox block (two Box-Muller pairs).
inline void normals4(const Stream& s, uint64_t blk, float z[4]) {
  const Block4 b = s.block(blk);
  for (int p = 0; p < 2; ++p) {
    const float u1 = u01(b.v[2 * p]);
    const float u2 = u01(b.v[2 * p + 1]);
    const float r = std::sqrt(-2.0f * std::log(u1));
    const float th = 6.2831853071795864769f * u2;
    z[2 * p] = r * std::cos(th);
    z[2 * p + 1] = r * std::sin(th);
  }
}

// Element i of the N(mean, std) stream (seed, tag).
inline float normal_at(const Stream& s, uint64_t i, float mean, float stdv) {
  float z[4];
  normals4(s, i >> 2, z);
  return mean + stdv * z[i & 3];
}

// Fill out[0..n) with elements first..first+n of the stream; n need not be a
// multiple of 4.
inline void normal_span(const Stream& s, uint64_t first, uint64_t n, float mean, float stdv,
                        float* out) {
  uint64_t i = first;
  const uint64_t end = first + n;
  while (i < end) {
    float z[4];
    normals4(s, i >> 2, z);
    for (uint64_t j = i & 3; j < 4 && i < end; ++j, ++i) out[i - first] = mean + stdv * z[j];
  }
}

inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u) return uint16_t((u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u));
  u += 0x7FFFu + ((u >> 16) & 1u);
  return uint16_t(u >> 16);
}

template <class F>
void parallel_rows(int64_t rows, int threads, F&& fn) {
  if (threads <= 0) threads = int(std::max(1u, std::thread::hardware_concurrency()));
  if (rows < 2 || threads == 1) {
    fn(int64_t(0), rows);
    return;
  }
  threads = int(std::min<int64_t>(threads, rows));
  std::vector<std::thread> pool;
  pool.reserve(threads);
  const int64_t chunk = (rows + threads - 1) / threads;
  for (int t = 0; t < threads; ++t) {
    const int64_t a = t * chunk, b = std::min(rows, a + chunk);
    if (a >= b) break;
    pool.emplace_back([&fn, a, b] { fn(a, b); });
  }
  for (auto& th : pool) th.join();
}

// Nearest E2M1 magnitude code for a >= 0 (ties to the even code, saturating).
// Decision points are the midpoints between neighbouring magnitudes
// {0, .5, 1, 1.5, 2, 3, 4, 6}: 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5. At a tie
// the code with a zero mantissa bit (even code) wins.
inline uint8_t e2m1_magnitude_code(float a) {
  if (a <= 0.25f) return 0;
  if (a < 0.75f) return 1;
  if (a <= 1.25f) return 2;
  if (a < 1.75f) return 3;
  if (a <= 2.5f) return 4;
  if (a < 3.5f) return 5;
  if (a <= 5.0f) return 6;
  return 7;
}

// Quantise one block of 32 fp32 values: returns the E8M0 byte, writes 16
// packed code bytes.
inline uint8_t quantize_block32(const float* v, uint8_t* packed) {
  float amax = 0.0f;
  for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs(v[i]));
  if (!(amax > 0.0f)) {
    std::memset(packed, 0, 16);
    return 0;
  }
  int ex = 0;
  std::frexp(amax, &ex);          // amax = m * 2^ex, m in [0.5, 1)
  int X = (ex - 1) - 2;           // floor(log2(amax)) - 2
  int e = std::min(254, std::max(0, X + 127));
  X = e - 127;
  for (int i = 0; i < 16; ++i) {
    uint8_t c[2];
    for (int h = 0; h < 2; ++h) {
      const float x = v[2 * i + h];
      const float t = std::ldexp(x, -X);
      uint8_t code = e2m1_magnitude_code(std::fabs(t));
      if (std::signbit(x)) code |= 8;
      c[h] = code;
    }
    packed[i] = uint8_t(c[0] | (c[1] << 4));
  }
  return uint8_t(e);
}

inline void quantize_int8_row(const float* w, int64_t K, int8_t* q, float* scale) {
  float amax = 0.0f;
  for (int64_t k = 0; k < K; ++k) amax = std::max(amax, std::fabs(w[k]));
  if (!(amax > 0.0f)) {
    *scale = 1.0f;
    std::memset(q, 0, size_t(K));
    return;
  }
  const float s = amax / 127.0f;
  *scale = s;
  for (int64_t k = 0; k < K; ++k) {
    float r = std::nearbyint(w[k] / s);
    r = std::min(127.0f, std::max(-127.0f, r));
    q[k] = int8_t(r);
  }
}

}  // namespace

extern "C" {

int v4in_version() { return 1; }

void v4in_philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3, uint32_t k0, uint32_t k1,
                        uint32_t* out4) {
  const Block4 b = philox4x32_10(c0, c1, c2, c3, k0, k1);
  for (int i = 0; i < 4; ++i) out4[i] = b.v[i];
}

// N(mean, std) fp32 values, elements [first, first+n) of stream (seed, tag).
void v4in_normal_f32(uint64_t seed, uint32_t tag, uint64_t first, uint64_t n, float mean, float stdv,
                     float* out, int threads) {
  const Stream s(seed, tag);
  const int64_t chunk = 1 << 16;
  const int64_t nchunks = int64_t((n + chunk - 1) / chunk);
  parallel_rows(nchunks, threads, [&](int64_t a, int64_t b) {
    for (int64_t c = a; c < b; ++c) {
      const uint64_t lo = uint64_t(c) * chunk;
      const uint64_t cnt = std::min<uint64_t>(chunk, n - lo);
      normal_span(s, first + lo, cnt, mean, stdv, out + lo);
    }
  });
}

// Same stream rounded to bf16 (bit patterns).
void v4in_normal_bf16(uint64_t seed, uint32_t tag, uint64_t first, uint64_t n, float mean, float stdv,
                      uint16_t* out, int threads) {
  const Stream s(seed, tag);
  const int64_t chunk = 1 << 16;
  const int64_t nchunks = int64_t((n + chunk - 1) / chunk);
  parallel_rows(nchunks, threads, [&](int64_t a, int64_t b) {
    std::vector<float> tmp(chunk);
    for (int64_t c = a; c < b; ++c) {
      const uint64_t lo = uint64_t(c) * chunk;
      const uint64_t cnt = std::min<uint64_t>(chunk, n - lo);
      normal_span(s, first + lo, cnt, mean, stdv, tmp.data());
      for (uint64_t i = 0; i < cnt; ++i) out[lo + i] = f32_to_bf16_rne(tmp[i]);
    }
  });
}

void v4in_f32_to_bf16(const float* in, uint64_t n, uint16_t* out) {
  for (uint64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}

// MXFP4-quantise given fp32 rows [rows, K] (K % 32 == 0): codes [rows, K/2],
// scales [rows, K/32].
int v4in_quantize_mxfp4(const float* w, int64_t rows, int64_t K, uint8_t* codes, uint8_t* scales,
                        int threads) {
  if (K % 32 != 0) return 1;
  parallel_rows(rows, threads, [&](int64_t a, int64_t b) {
    for (int64_t r = a; r < b; ++r)
      for (int64_t g = 0; g < K / 32; ++g)
        scales[r * (K / 32) + g] = quantize_block32(w + r * K + g * 32, codes + r * (K / 2) + g * 16);
  });
  return 0;
}

// Draw N(0, std) weights for a [rows, K] tensor (element index row*K + k of
// stream (seed, tag), rows counted from row0) and MXFP4-quantise them.
int v4in_mxfp4_normal(uint64_t seed, uint32_t tag, int64_t row0, int64_t rows, int64_t K, float stdv,
                      uint8_t* codes, uint8_t* scales, int threads) {
  if (K % 32 != 0) return 1;
  const Stream s(seed, tag);
  parallel_rows(rows, threads, [&](int64_t a, int64_t b) {
    std::vector<float> row(static_cast<size_t>(K));
    for (int64_t r = a; r < b; ++r) {
      normal_span(s, uint64_t(row0 + r) * uint64_t(K), uint64_t(K), 0.0f, stdv, row.data());
      for (int64_t g = 0; g < K / 32; ++g)
        scales[r * (K / 32) + g] = quantize_block32(row.data() + g * 32, codes + r * (K / 2) + g * 16);
    }
  });
  return 0;
}

int v4in_quantize_int8(const float* w, int64_t rows, int64_t K, int8_t* q, float* scale, int threads) {
  parallel_rows(rows, threads, [&](int64_t a, int64_t b) {
    for (int64_t r = a; r < b; ++r) quantize_int8_row(w + r * K, K, q + r * K, scale + r);
  });
  return 0;
}

int v4in_int8_normal(uint64_t seed, uint32_t tag, int64_t rows, int64_t K, float stdv, int8_t* q,
                     float* scale, int threads) {
  const Stream s(seed, tag);
  parallel_rows(rows, threads, [&](int64_t a, int64_t b) {
    std::vector<float> row(static_cast<size_t>(K));
    for (int64_t r = a; r < b; ++r) {
      normal_span(s, uint64_t(r) * uint64_t(K), uint64_t(K), 0.0f, stdv, row.data());
      quantize_int8_row(row.data(), K, q + r * K, scale + r);
    }
  });
  return 0;
}

// Zipf(s) over ranks 1..vocab, n draws; out[i] = rank - 1.
int v4in_zipf_ids(uint64_t seed, uint32_t tag, int64_t n, int64_t vocab, double s, int32_t* out,
                  int threads) {
  if (vocab <= 0) return 1;
  std::vector<double> cdf(static_cast<size_t>(vocab));
  double acc = 0.0;
  for (int64_t r = 1; r <= vocab; ++r) {
    acc += std::pow(double(r), -s);
    cdf[size_t(r - 1)] = acc;
  }
  for (auto& c : cdf) c /= acc;
  cdf.back() = 1.0;
  const Stream st(seed, tag);
  parallel_rows(n, threads, [&](int64_t a, int64_t b) {
    for (int64_t i = a; i < b; ++i) {
      const Block4 blk = st.block(uint64_t(i));
      // 53-bit uniform in [0, 1).
      const uint64_t bits = (uint64_t(blk.v[0]) << 21) ^ uint64_t(blk.v[1] >> 11);
      const double u = double(bits & ((uint64_t(1) << 53) - 1)) * (1.0 / 9007199254740992.0);
      // smallest r with cdf[r] > u
      const auto it = std::upper_bound(cdf.begin(), cdf.end(), u);
      int64_t idx = int64_t(it - cdf.begin());
      if (idx >= vocab) idx = vocab - 1;
      out[i] = int32_t(idx);
    }
  });
  return 0;
}

// tid2eid [vocab, k]: row v holds k distinct experts drawn by a partial
// Fisher-Yates shuffle of 0..E-1 (draw j uses lane j%4 of Philox block
// (v, sub=j/4)).
int v4in_tid2eid(uint64_t seed, uint32_t tag, int64_t vocab, int32_t k, int32_t E, int32_t* out,
                 int threads) {
  if (k > E || k <= 0) return 1;
  const Stream st(seed, tag);
  parallel_rows(vocab, threads, [&](int64_t a, int64_t b) {
    std::vector<int32_t> perm(static_cast<size_t>(E));
    for (int64_t v = a; v < b; ++v) {
      for (int32_t e = 0; e < E; ++e) perm[size_t(e)] = e;
      Block4 blk{};
      for (int32_t j = 0; j < k; ++j) {
        if ((j & 3) == 0) blk = st.block(uint64_t(v), uint32_t(j >> 2));
        const uint32_t r = blk.v[j & 3];
        const int32_t span = E - j;
        const int32_t pick = j + int32_t((uint64_t(r) * uint64_t(span)) >> 32);
        std::swap(perm[size_t(j)], perm[size_t(pick)]);
        out[v * k + j] = perm[size_t(j)];
      }
    }
  });
  return 0;
}

}  // extern "C"
