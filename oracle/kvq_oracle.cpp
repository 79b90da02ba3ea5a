// kvq_oracle.cpp — plain, slow CPU oracle for the asymmetric low-bit KV cache and decode attention.
//
// TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call this file; only the
// tests, the smoke check and the CPU-baseline leg of the benchmark do. It shares no code, header,
// table or helper with the CUDA library: every step below is written out again from its definition.
//
// What it computes, and the passages it follows:
//  * Keys are quantized per channel and values per token (The Asymmetric Key-Value Cache Compression
//    framework page, Method; KVQuant review, Method and Key idea; KV cache quantization wiki page,
//    verification notes on the KIVI full text: key outliers sit in a few fixed channels, and per-token
//    value quantization keeps each token's error to itself).
//  * Keys are grouped every G tokens along the sequence; the grouped part and a full-precision
//    residual part both enter the attention score; freshly quantized groups are appended along the
//    token axis (KV cache quantization wiki page, verification notes, KIVI grouped/residual split).
//  * The newest tokens stay in FP16 (framework page, In practice: a window of 32 to 128 tokens).
//  * Optional Walsh-Hadamard rotation of keys, with the same orthogonal transform applied to the
//    query so q.k is unchanged (framework page, Method and In practice; Dual-QK abstract on the
//    thelatestinai listing).
//  * Min/max scale and zero-point, round to nearest, 2 or 4 bits (KVQuant review, Problem: 2 bits
//    give 4 levels; uniform INT4/INT3/INT2 grids in Comparison).
//  * Decode attention is one query against every cached token (NOVA-KV abstract on the
//    thelatestinai listing: each decoding step reads the whole cache).
//
// Readings where the pages are silent (each also listed in the design notes):
//  R1  quantized length Q = G * floor(max(T - R, 0) / G); tokens [Q, T) are the FP16 residual,
//      kept in a ring of R + G slots at slot t mod (R + G).
//  R2  Hadamard: Sylvester order H[i][j] = (-1)^popcount(i & j), fp32 butterfly with strides
//      1, 2, ..., 64 (pair (i, i+h) -> (a+b, a-b)), then multiply by fp32(1/sqrt(128)), then round
//      to fp16 (keys). The query gets the same rotation in fp64 here.
//  R3  group min/max under the IEEE total order with -0 < +0.
//  R4  s32 = (f32(mx) - f32(mn)) / f32(2^b - 1); s16 = fp16_rn(s32); zero = mn (fp16).
//  R5  s16 == 0 -> all codes 0; else inv = 1 / f32(s16),
//      code = clamp(rint_half_even((f32(x) - f32(mn)) * inv), 0, 2^b - 1), each op one IEEE fp32
//      rounding, never fused.
//  R6  dequant x^ = code * s16 + zero, evaluated here in fp64.
//  R7  attention in fp64: no causal mask; softmax over all T tokens (the sink token, R10, and RoPE,
//      R11, are options, off by default).
//  R8  packed layouts "tile v1" (mma fragment order) and "rows v2" (one token's key codes, one
//      channel's value codes per row); see key_word_bit / value_word_bit / key_param_pos and the
//      v2 functions below.
//  R10 optional attention sink: the first token stays in fp16 (see quantize_span and key_row).
//  R11 optional pre-RoPE keys (rope_theta > 0; KVQuant review, Method and Key idea: keys are
//      quantized before RoPE, and RoPE is applied after dequantization). The cache holds the keys as
//      given, without RoPE; decode rotates every key at its absolute position t (0-based) after
//      dequantization, or from its fp16 row: channel pairs (i, i + 64), i < 64, by the angle
//      t * theta^(-i/64), k'[i] = k[i] cos - k[i+64] sin, k'[i+64] = k[i] sin + k[i+64] cos, in
//      fp64. The query is taken as given (rotated at its own position by the caller). RoPE and the
//      Hadamard option exclude each other.
//  R12 optional dense-and-sparse outliers (outliers = 1; KVQuant review, Method: per-vector
//      thresholds move about 1% of the entries into an fp16 sparse store). Per quantized token and
//      tensor, the entry of largest magnitude (ties: the lowest channel) is that vector's outlier,
//      1 of 128 entries. It is kept exactly in fp16 (channel and value per token), left out of the
//      min/max of its key group (per channel) or value group (per token), and coded 0; dequantization
//      puts the fp16 value back. A key channel whose entries in a group are all outliers gets scale
//      and zero 0. The sink token (R10) has no outlier; the fp16 window needs none.
//  R13 optional paged storage (page_tokens = P > 0; KVQuant review, Limitations, Future work and
//      Sparks: blocked allocation instead of copying the previous tokens' data on every update).
//      The quantized part of a unit is cut into logical pages of P tokens (P a multiple of 128, so
//      a page holds whole 16-token tiles, whole 128-token value blocks of rows v2 and whole key
//      groups). Logical page j of a unit lives in physical page page_table[unit][j] of a pool of
//      num_pages pages; a page holds exactly what the contiguous layout holds for its P tokens
//      (codes, key group scale / zero, value scale / zero, outliers), at the in-page token t mod P.
//      The fp16 window and the sink row stay per unit. Paging changes addresses only, never values.
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fno-fast-math -fPIC -shared (x86-64 SSE scalar fp32).

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>
#include <algorithm>

namespace {

// ------------------------------------------------------------------------------------------------
// IEEE 754 binary16 <-> binary32, written from the format definition (1 sign, 5 exponent bits with
// bias 15, 10 fraction bits; subnormals have value fraction * 2^-24).
// ------------------------------------------------------------------------------------------------
float half_to_float(uint16_t h) {
  const uint32_t sign = h >> 15, expo = (h >> 10) & 0x1fu, frac = h & 0x3ffu;
  float mag;
  if (expo == 0) {
    mag = std::ldexp(static_cast<float>(frac), -24);  // exact: frac < 2^10
  } else if (expo == 31) {
    mag = frac ? std::nanf("") : INFINITY;
  } else {
    mag = std::ldexp(static_cast<float>(frac | 0x400u), static_cast<int>(expo) - 25);  // exact
  }
  return sign ? -mag : mag;
}

// Round-to-nearest-even conversion of a binary32 to binary16, done on the integer significand.
uint16_t float_to_half(float f) {
  uint32_t x;
  std::memcpy(&x, &f, 4);
  const uint16_t sign = static_cast<uint16_t>((x >> 16) & 0x8000u);
  const uint32_t ax = x & 0x7fffffffu;
  if (ax > 0x7f800000u) return sign | 0x7e00u;  // NaN
  if (ax == 0x7f800000u) return sign | 0x7c00u;  // infinity
  const int e = static_cast<int>(ax >> 23) - 127;  // unbiased exponent (normal binary32)
  uint32_t sig = (ax & 0x7fffffu) | (ax >= 0x00800000u ? 0x800000u : 0u);  // 24-bit significand
  int e_eff = (ax >= 0x00800000u) ? e : -126;  // binary32 subnormals: value = sig * 2^-149
  // value = sig * 2^(e_eff - 23). Target unit: fp16 normal with exponent E has ulp 2^(E-10);
  // subnormal ulp 2^-24. Choose the ulp of the result, shift the significand to it, round.
  int target_exp = std::max(e_eff, -14);  // exponent whose ulp we round to
  int shift = target_exp - 10 - (e_eff - 23);  // bits to drop from sig
  // shift >= 32 means the magnitude is below 2^-32, far under half the smallest subnormal: zero.
  if (shift >= 32) return sign;
  uint32_t q = sig >> shift;
  const uint32_t rem = sig & ((1u << shift) - 1u);
  const uint32_t half = 1u << (shift - 1);
  if (rem > half || (rem == half && (q & 1u))) q += 1;
  // q is the significand in units of the result ulp. Rebuild the binary16 bit pattern.
  uint32_t out;
  if (target_exp == -14 && q < 0x400u) {
    out = q;  // subnormal (or zero)
  } else {
    // q in [2^10, 2^11] for a normal; a carry to 2^11 bumps the exponent.
    int E = target_exp;
    if (q >= 0x800u) { q >>= 1; E += 1; }
    if (E > 15) return sign | 0x7c00u;  // overflow -> infinity
    out = (static_cast<uint32_t>(E + 15) << 10) | (q & 0x3ffu);
  }
  return static_cast<uint16_t>(sign | out);
}

// IEEE 754-2019 minimum / maximum on non-NaN binary16, with -0 ordered below +0 (reading R3).
inline uint32_t order_key(uint16_t h) { return (h & 0x8000u) ? (~h & 0xffffu) : (h | 0x8000u); }
inline uint16_t hmin(uint16_t a, uint16_t b) { return order_key(b) < order_key(a) ? b : a; }
inline uint16_t hmax(uint16_t a, uint16_t b) { return order_key(b) > order_key(a) ? b : a; }

// fp32 value of 1/sqrt(128) rounded to nearest (bit pattern 0x3DB504F3).
float inv_sqrt128_f32() {
  const uint32_t bits = 0x3DB504F3u;
  float f;
  std::memcpy(&f, &bits, 4);
  return f;
}

// Walsh-Hadamard rotation of one 128-vector in fp32 (reading R2). Stride-h butterflies in the order
// h = 1, 2, 4, ..., 64; each pair (i, i+h) with (i & h) == 0 becomes (a + b, a - b); then every
// entry is multiplied by fp32(1/sqrt(128)).
void wht128_f32(float* x) {
  for (int h = 1; h < 128; h <<= 1)
    for (int i = 0; i < 128; ++i)
      if ((i & h) == 0) {
        const float a = x[i], b = x[i + h];
        x[i] = a + b;
        x[i + h] = a - b;
      }
  const float s = inv_sqrt128_f32();
  for (int i = 0; i < 128; ++i) x[i] = x[i] * s;
}

// The same rotation in fp64 with the exact scale 1/sqrt(128) (used for the query, reading R2).
void wht128_f64(double* x) {
  for (int h = 1; h < 128; h <<= 1)
    for (int i = 0; i < 128; ++i)
      if ((i & h) == 0) {
        const double a = x[i], b = x[i + h];
        x[i] = a + b;
        x[i + h] = a - b;
      }
  const double s = 1.0 / std::sqrt(128.0);
  for (int i = 0; i < 128; ++i) x[i] *= s;
}

// ------------------------------------------------------------------------------------------------
// Asymmetric min/max quantizer of one group (readings R3-R5).
// ------------------------------------------------------------------------------------------------
struct GroupQ {
  uint16_t scale, zero;
};

// skip (optional): entries with skip[i * skip_stride] != 0 stay out of the min / max and get code 0
// (reading R12); a group with every entry skipped gets scale and zero 0.
GroupQ quantize_group(const uint16_t* x, int n, int stride, int bits, uint8_t* codes, int code_stride,
                      const uint8_t* skip = nullptr, int skip_stride = 0) {
  int first = 0;
  while (skip && first < n && skip[first * skip_stride]) ++first;
  if (first == n) {
    for (int i = 0; i < n; ++i) codes[i * code_stride] = 0;
    return GroupQ{0, 0};
  }
  uint16_t mn = x[first * stride], mx = x[first * stride];
  for (int i = first + 1; i < n; ++i) {
    if (skip && skip[i * skip_stride]) continue;
    mn = hmin(mn, x[i * stride]);
    mx = hmax(mx, x[i * stride]);
  }
  const float levels = static_cast<float>((1 << bits) - 1);
  const float range = half_to_float(mx) - half_to_float(mn);
  const float s32 = range / levels;
  const uint16_t s16 = float_to_half(s32);
  GroupQ g{s16, mn};
  if ((s16 & 0x7fffu) == 0) {
    for (int i = 0; i < n; ++i) codes[i * code_stride] = 0;
    return g;
  }
  const float inv = 1.0f / half_to_float(s16);
  const float zf = half_to_float(mn);
  const int top = (1 << bits) - 1;
  for (int i = 0; i < n; ++i) {
    if (skip && skip[i * skip_stride]) {
      codes[i * code_stride] = 0;
      continue;
    }
    const float d = half_to_float(x[i * stride]) - zf;
    const float v = d * inv;
    float r = std::nearbyint(v);  // default rounding mode: nearest, ties to even
    int c = static_cast<int>(r);
    if (c < 0) c = 0;
    if (c > top) c = top;
    codes[i * code_stride] = static_cast<uint8_t>(c);
  }
  return g;
}

// ------------------------------------------------------------------------------------------------
// Packed layout "tile v1" (reading R8). The cache of one (sequence, KV head) is cut into tiles of 16
// tokens x 128 channels. A tile holds 32 "lanes" of W = 2*bits u32 words (4 words at 2 bits, 8 at
// 4 bits); lane L's word w sits at word (w / 4) * 128 + 4 * L + (w % 4) of the tile. Each word holds
// P = 16 / bits code pairs: pair k has element e = 0 at bits [bits*k, bits*k + bits) and e = 1 at
// bits [16 + bits*k, ...). Pair slot p = w * P + k names (m = p / 4, reg = p % 4, u = reg % 2,
// h = reg / 2), and with L = 4 r + qd:
//   keys:   token i = r + 8u,          channel c = 16m + 2qd + 8h + e
//   values: token i = 2qd + 8h + e,    channel c = 16m + r + 8u
// Per-group key scale and zero store channel c = 16m + 2qd + 8h + e at position 32qd + 4m + 2h + e.
// Value scale and zero are [token][channel group] in natural order.
// ------------------------------------------------------------------------------------------------
inline void slot_to_word_bit(int lane, int p, int bits, int e, int* word, int* bit) {
  const int P = 16 / bits;
  const int w = p / P, k = p % P;
  *word = (w / 4) * 128 + 4 * lane + (w % 4);
  *bit = bits * k + 16 * e;
}

void key_word_bit(int i, int c, int bits, int* word, int* bit) {
  const int r = i % 8, u = i / 8;
  const int m = c / 16, within = c % 16;
  const int h = within / 8, qd = (within % 8) / 2, e = within % 2;
  const int lane = 4 * r + qd;
  const int p = 4 * m + (u + 2 * h);
  slot_to_word_bit(lane, p, bits, e, word, bit);
}

void value_word_bit(int i, int c, int bits, int* word, int* bit) {
  const int m = c / 16, within = c % 16;
  const int r = within % 8, u = within / 8;
  const int h = i / 8, qd = (i % 8) / 2, e = i % 2;
  const int lane = 4 * r + qd;
  const int p = 4 * m + (u + 2 * h);
  slot_to_word_bit(lane, p, bits, e, word, bit);
}

int key_param_pos(int c) {
  const int m = c / 16, within = c % 16;
  const int h = within / 8, qd = (within % 8) / 2, e = within % 2;
  return 32 * qd + 4 * m + 2 * h + e;
}

// Layout "rows v2". Keys: token t's codes form a row of 4*bits u32 words; channel pair j = c / 2
// sits in word j / P (P = 16 / bits pairs per word) as pair k = j % P: channel 2j at bits
// [bits*k, bits*k + bits), channel 2j + 1 at bits [16 + bits*k, ...). Values: tokens are cut into
// blocks of 128; within a block, channel c's codes form a row of 4*bits words and token pair
// j = i / 2 (i = t % 128) sits in word j / P as pair k = j % P (token 2j low, 2j + 1 high).
// Key scale / zero keep the natural channel order.
void key_word_bit_v2(int64_t t, int c, int bits, int64_t* word, int* bit) {
  const int P = 16 / bits;
  const int j = c / 2, e = c % 2;
  *word = t * (4 * bits) + j / P;
  *bit = bits * (j % P) + 16 * e;
}

void value_word_bit_v2(int64_t t, int c, int bits, int64_t* word, int* bit) {
  const int P = 16 / bits;
  const int64_t block = t / 128;
  const int i = static_cast<int>(t % 128);
  const int j = i / 2, e = i % 2;
  *word = (block * 128 + c) * (4 * bits) + j / P;
  *bit = bits * (j % P) + 16 * e;
}

}  // namespace

// ================================================================================================
// C interface (host pointers only).
// ================================================================================================
extern "C" {

typedef struct {
  int32_t batch, num_q_heads, num_kv_heads, head_dim;
  int32_t key_bits, value_bits, group_size, residual, hadamard, layout;  // layout: 1 = tile v1, 2 = rows v2
  int32_t sink;        // 1: the first token stays in fp16 (reading R10)
  float rope_theta;    // > 0: keys are cached before RoPE, decode applies it (reading R11); 0: off
  int32_t outliers;    // 1: each quantized token's largest-magnitude key and value entry stay fp16 (R12)
  int32_t page_tokens; // > 0: paged storage with pages of this many tokens (reading R13); 0: contiguous
  int32_t num_pages;   // pages in the pool (paged storage only)
  int64_t capacity;    // tokens per sequence (paged: capacity / page_tokens logical pages per unit)
} kvq_ref_config;

// Contiguous storage: every per-token array below has one slot of capacity tokens per unit
// ([B][Hkv][...]). Paged storage (R13): one slot of page_tokens tokens per physical page
// ([num_pages][...]); the ring stays [B][Hkv][...].
typedef struct {
  uint32_t* k_codes;  // [B][Hkv][Cap/16][64*key_bits]
  uint32_t* v_codes;  // [B][Hkv][Cap/16][64*value_bits]
  uint16_t* k_scale;  // [B][Hkv][Cap/G][128] (permuted channel order)
  uint16_t* k_zero;   // same
  uint16_t* v_scale;  // [B][Hkv][Cap][128/G]
  uint16_t* v_zero;   // same
  uint16_t* k_res;    // [B][Hkv][R+G+sink][128] ring, fp16 (row R+G: the first token when sink is on)
  uint16_t* v_res;    // same
  int64_t* seq_len;   // [B]
  uint16_t* k_out_ch;   // [B][Hkv][Cap] channel of the token's key outlier (0xffff: none); reading R12
  uint16_t* k_out_val;  // [B][Hkv][Cap] its fp16 value
  uint16_t* v_out_ch;   // same for values
  uint16_t* v_out_val;
  int32_t* page_table;  // [B][Hkv][Cap/page_tokens] physical page of each logical page (paged only)
} kvq_ref_cache;

enum { REF_OK = 0, REF_ERR_ARG = -1, REF_ERR_CAPACITY = -3 };

static int check_config(const kvq_ref_config* c) {
  if (!c) return REF_ERR_ARG;
  if (c->head_dim != 128) return REF_ERR_ARG;
  if (c->batch < 0 || c->num_kv_heads <= 0 || c->num_q_heads <= 0) return REF_ERR_ARG;
  if (c->num_q_heads % c->num_kv_heads) return REF_ERR_ARG;
  if ((c->key_bits != 2 && c->key_bits != 4) || (c->value_bits != 2 && c->value_bits != 4)) return REF_ERR_ARG;
  const int G = c->group_size;
  if (G <= 0 || G % 16 || 128 % G) return REF_ERR_ARG;
  if (c->residual < 0 || c->capacity < 0 || c->capacity % G) return REF_ERR_ARG;
  if (c->layout != 1 && c->layout != 2) return REF_ERR_ARG;
  if (c->sink != 0 && c->sink != 1) return REF_ERR_ARG;
  if (!(c->rope_theta >= 0.0f) || !std::isfinite(c->rope_theta)) return REF_ERR_ARG;
  if (c->rope_theta > 0.0f && c->hadamard) return REF_ERR_ARG;
  if (c->outliers != 0 && c->outliers != 1) return REF_ERR_ARG;
  if (c->page_tokens < 0 || c->num_pages < 0) return REF_ERR_ARG;
  if (c->page_tokens > 0 && (c->page_tokens % 128 || c->capacity % c->page_tokens)) return REF_ERR_ARG;
  return REF_OK;
}

static int64_t quantized_len(int64_t T, int R, int G) {
  const int64_t over = T - R;
  return over > 0 ? (over / G) * G : 0;
}

// Word (within the unit's code buffer) and bit of the code of token t, channel ch, per layout.
static void key_pos(const kvq_ref_config* c, int64_t t, int ch, int64_t* word, int* bit) {
  if (c->layout == 2) {
    key_word_bit_v2(t, ch, c->key_bits, word, bit);
  } else {
    int w;
    key_word_bit(static_cast<int>(t % 16), ch, c->key_bits, &w, bit);
    *word = (t / 16) * (64 * c->key_bits) + w;
  }
}
static void value_pos(const kvq_ref_config* c, int64_t t, int ch, int64_t* word, int* bit) {
  if (c->layout == 2) {
    value_word_bit_v2(t, ch, c->value_bits, word, bit);
  } else {
    int w;
    value_word_bit(static_cast<int>(t % 16), ch, c->value_bits, &w, bit);
    *word = (t / 16) * (64 * c->value_bits) + w;
  }
}
static int key_param_index(const kvq_ref_config* c, int ch) { return c->layout == 2 ? ch : key_param_pos(ch); }

struct Dims {
  int64_t slot_tokens;                                 // tokens per storage slot: capacity (contiguous) or page_tokens (R13)
  int64_t kw_tile, vw_tile, tiles, groups, ring, vpt;  // words per tile, tiles/slot, groups/slot, ring slots, value groups per token
  int64_t kwords, vwords;                              // code words per slot
  int64_t res_rows;                                    // rows of k_res / v_res per unit: ring slots + the sink row
};
static Dims dims(const kvq_ref_config* c) {
  Dims d;
  d.kw_tile = 64 * c->key_bits;
  d.vw_tile = 64 * c->value_bits;
  d.slot_tokens = c->page_tokens > 0 ? c->page_tokens : c->capacity;
  d.tiles = d.slot_tokens / 16;
  d.kwords = d.slot_tokens * 4 * c->key_bits;
  d.vwords = (c->layout == 2 ? (d.slot_tokens + 127) / 128 * 128 : d.slot_tokens) * 4 * c->value_bits;
  d.groups = d.slot_tokens / c->group_size;
  d.ring = c->residual + c->group_size;
  d.res_rows = d.ring + c->sink;
  d.vpt = 128 / c->group_size;
  return d;
}

// Storage slot of token t of `unit` and the token's index within it (reading R13): the unit and t
// for contiguous storage; the physical page of logical page t / P and t mod P for paged storage.
static void locate(const kvq_ref_config* c, const kvq_ref_cache* cache, int64_t unit, int64_t t, int64_t* slot,
                   int64_t* ts) {
  if (c->page_tokens == 0) {
    *slot = unit;
    *ts = t;
    return;
  }
  const int64_t pages_per_unit = c->capacity / c->page_tokens;
  *slot = cache->page_table[unit * pages_per_unit + t / c->page_tokens];
  *ts = t % c->page_tokens;
}

// Whether every logical page holding tokens [0, n) of `unit` maps to a page of the pool.
static bool pages_valid(const kvq_ref_config* c, const kvq_ref_cache* cache, int64_t unit, int64_t n) {
  if (c->page_tokens == 0) return true;
  const int64_t pages_per_unit = c->capacity / c->page_tokens;
  for (int64_t j = 0; j * c->page_tokens < n; ++j) {
    const int32_t p = cache->page_table[unit * pages_per_unit + j];
    if (p < 0 || p >= c->num_pages) return false;
  }
  return true;
}

// The channel of a token vector's largest-magnitude entry (reading R12): binary16 magnitudes order
// like the integers of their low 15 bits (non-NaN); ties go to the lowest channel.
static int largest_entry(const uint16_t* x) {
  int best = 0;
  for (int ch = 1; ch < 128; ++ch)
    if ((x[ch] & 0x7fffu) > (x[best] & 0x7fffu)) best = ch;
  return best;
}

// Quantize tokens [t0, t0 + G) of key unit `kt` (fp16 [T][128], already rotated if enabled) into key
// group t0 / G, and the same tokens of value unit `vt` per token.
// With the sink on (reading R10) the first token of the sequence stays out of the quantizer: key group
// 0's min/max run over its other G - 1 tokens, and the first token's key codes, value codes, value
// scale and value zero are 0 (it is read from its fp16 row instead).
static void quantize_span(const kvq_ref_config* c, const kvq_ref_cache* cache, int64_t unit, int64_t t0,
                          const uint16_t* kt, int64_t k_ld, const uint16_t* vt, int64_t v_ld) {
  const Dims d = dims(c);
  const int G = c->group_size;
  const int skip = (c->sink && t0 == 0) ? 1 : 0;  // tokens at the start of the span kept out
  int64_t slot, ts0;  // where the span is stored (a group never crosses a page: P is a multiple of G)
  locate(c, cache, unit, t0, &slot, &ts0);
  // Outliers (reading R12): each token's largest-magnitude key entry and value entry.
  std::vector<uint8_t> kout(static_cast<size_t>(G) * 128, 0), vout(static_cast<size_t>(G) * 128, 0);
  if (c->outliers) {
    for (int i = 0; i < G; ++i) {
      const int64_t at = slot * d.slot_tokens + ts0 + i;
      if (i < skip) {  // the sink token is fp16 as a whole
        cache->k_out_ch[at] = cache->v_out_ch[at] = 0xffffu;
        cache->k_out_val[at] = cache->v_out_val[at] = 0;
        continue;
      }
      const int kch = largest_entry(kt + i * k_ld), vch = largest_entry(vt + i * v_ld);
      kout[i * 128 + kch] = 1;
      vout[i * 128 + vch] = 1;
      cache->k_out_ch[at] = static_cast<uint16_t>(kch);
      cache->k_out_val[at] = kt[i * k_ld + kch];
      cache->v_out_ch[at] = static_cast<uint16_t>(vch);
      cache->v_out_val[at] = vt[i * v_ld + vch];
    }
  }
  // Keys: per channel over the G (or G - 1) tokens of the group, outliers left out.
  std::vector<uint8_t> kc(static_cast<size_t>(G) * 128, 0);
  const int64_t g = ts0 / G;
  for (int ch = 0; ch < 128; ++ch) {
    GroupQ q = quantize_group(kt + skip * k_ld + ch, G - skip, static_cast<int>(k_ld), c->key_bits,
                              kc.data() + skip * 128 + ch, 128, kout.data() + skip * 128 + ch, 128);
    const int pos = key_param_index(c, ch);
    cache->k_scale[(slot * d.groups + g) * 128 + pos] = q.scale;
    cache->k_zero[(slot * d.groups + g) * 128 + pos] = q.zero;
  }
  uint32_t* kbuf = cache->k_codes + slot * d.kwords;
  for (int i = 0; i < G; ++i) {
    const int64_t t = ts0 + i;
    for (int ch = 0; ch < 128; ++ch) {
      int64_t word;
      int bit;
      key_pos(c, t, ch, &word, &bit);
      const uint32_t mask = ((1u << c->key_bits) - 1u) << bit;
      kbuf[word] = (kbuf[word] & ~mask) | (static_cast<uint32_t>(kc[i * 128 + ch]) << bit);
    }
  }
  // Values: per token over channel groups of G.
  std::vector<uint8_t> vc(128);
  for (int i = 0; i < G; ++i) {
    const int64_t t = ts0 + i;
    for (int j = 0; j < d.vpt; ++j) {
      GroupQ q{0, 0};
      if (i < skip)
        std::memset(vc.data() + j * G, 0, G);
      else
        q = quantize_group(vt + i * v_ld + j * G, G, 1, c->value_bits, vc.data() + j * G, 1,
                           vout.data() + i * 128 + j * G, 1);
      cache->v_scale[(slot * d.slot_tokens + t) * d.vpt + j] = q.scale;
      cache->v_zero[(slot * d.slot_tokens + t) * d.vpt + j] = q.zero;
    }
    uint32_t* vbuf = cache->v_codes + slot * d.vwords;
    for (int ch = 0; ch < 128; ++ch) {
      int64_t word;
      int bit;
      value_pos(c, t, ch, &word, &bit);
      const uint32_t mask = ((1u << c->value_bits) - 1u) << bit;
      vbuf[word] = (vbuf[word] & ~mask) | (static_cast<uint32_t>(vc[ch]) << bit);
    }
  }
}

static void rotate_key_f16(const uint16_t* in, uint16_t* out) {
  float x[128];
  for (int i = 0; i < 128; ++i) x[i] = half_to_float(in[i]);
  wht128_f32(x);
  for (int i = 0; i < 128; ++i) out[i] = float_to_half(x[i]);
}

static void prefill_unit(const kvq_ref_config* c, kvq_ref_cache* cache, const uint16_t* k, const uint16_t* v,
                         int64_t sb, int64_t st, int64_t sh, int64_t b, int64_t kvh, int64_t T) {
  const Dims d = dims(c);
  const int G = c->group_size;
  const int64_t unit = b * c->num_kv_heads + kvh;
  const int64_t Q = quantized_len(T, c->residual, G);
  // Gather this unit's tokens into contiguous [T][128] (keys rotated when enabled).
  std::vector<uint16_t> kt(static_cast<size_t>(T) * 128), vt(static_cast<size_t>(T) * 128);
  for (int64_t t = 0; t < T; ++t) {
    const uint16_t* ks = k + b * sb + t * st + kvh * sh;
    const uint16_t* vs = v + b * sb + t * st + kvh * sh;
    if (c->hadamard)
      rotate_key_f16(ks, &kt[t * 128]);
    else
      std::memcpy(&kt[t * 128], ks, 256);
    std::memcpy(&vt[t * 128], vs, 256);
  }
  for (int64_t t0 = 0; t0 < Q; t0 += G) quantize_span(c, cache, unit, t0, &kt[t0 * 128], 128, &vt[t0 * 128], 128);
  for (int64_t t = Q; t < T; ++t) {
    const int64_t slot = t % d.ring;
    std::memcpy(cache->k_res + (unit * d.res_rows + slot) * 128, &kt[t * 128], 256);
    std::memcpy(cache->v_res + (unit * d.res_rows + slot) * 128, &vt[t * 128], 256);
  }
  if (c->sink && T > 0) {  // the first token's fp16 row (reading R10)
    std::memcpy(cache->k_res + (unit * d.res_rows + d.ring) * 128, &kt[0], 256);
    std::memcpy(cache->v_res + (unit * d.res_rows + d.ring) * 128, &vt[0], 256);
  }
}

// Prefill: quantize the first Q_b tokens of every (sequence, KV head) and keep [Q_b, T_b) in FP16.
// k, v: fp16 [b][t][h][d] with element strides (sb, st, sh); d contiguous.
int kvq_ref_quantize_prefill(const kvq_ref_config* c, kvq_ref_cache* cache, const uint16_t* k, const uint16_t* v,
                             int64_t sb, int64_t st, int64_t sh, const int64_t* seq_lens, int nthreads) {
  int rc = check_config(c);
  if (rc) return rc;
  for (int b = 0; b < c->batch; ++b)
    if (seq_lens[b] < 0 || seq_lens[b] > c->capacity) return REF_ERR_CAPACITY;
  const int64_t units = static_cast<int64_t>(c->batch) * c->num_kv_heads;
  for (int64_t u = 0; u < units; ++u)
    if (!pages_valid(c, cache, u, quantized_len(seq_lens[u / c->num_kv_heads], c->residual, c->group_size)))
      return REF_ERR_ARG;
  auto work = [&](int64_t u0, int64_t step) {
    for (int64_t u = u0; u < units; u += step) {
      const int64_t b = u / c->num_kv_heads, h = u % c->num_kv_heads;
      prefill_unit(c, cache, k, v, sb, st, sh, b, h, seq_lens[b]);
    }
  };
  if (nthreads <= 1) {
    work(0, 1);
  } else {
    std::vector<std::thread> pool;
    for (int i = 0; i < nthreads; ++i) pool.emplace_back(work, i, nthreads);
    for (auto& t : pool) t.join();
  }
  for (int b = 0; b < c->batch; ++b) cache->seq_len[b] = seq_lens[b];
  return REF_OK;
}

// Append one token to every sequence; flush a key/value group when the residual window has grown
// past R by a whole group. k_new, v_new: fp16 [B][Hkv][128].
int kvq_ref_append_token(const kvq_ref_config* c, kvq_ref_cache* cache, const uint16_t* k_new, const uint16_t* v_new) {
  int rc = check_config(c);
  if (rc) return rc;
  const Dims d = dims(c);
  const int G = c->group_size;
  for (int b = 0; b < c->batch; ++b)
    if (cache->seq_len[b] + 1 > c->capacity) return REF_ERR_CAPACITY;
  for (int b = 0; b < c->batch; ++b)
    for (int h = 0; h < c->num_kv_heads; ++h)
      if (!pages_valid(c, cache, static_cast<int64_t>(b) * c->num_kv_heads + h,
                       quantized_len(cache->seq_len[b] + 1, c->residual, G)))
        return REF_ERR_ARG;
  for (int b = 0; b < c->batch; ++b) {
    const int64_t t = cache->seq_len[b];
    const int64_t Q_old = quantized_len(t, c->residual, G);
    const int64_t Q_new = quantized_len(t + 1, c->residual, G);
    for (int h = 0; h < c->num_kv_heads; ++h) {
      const int64_t unit = static_cast<int64_t>(b) * c->num_kv_heads + h;
      const uint16_t* ks = k_new + unit * 128;
      const uint16_t* vs = v_new + unit * 128;
      const int64_t slot = t % d.ring;
      uint16_t* kslot = cache->k_res + (unit * d.res_rows + slot) * 128;
      uint16_t* vslot = cache->v_res + (unit * d.res_rows + slot) * 128;
      if (c->hadamard)
        rotate_key_f16(ks, kslot);
      else
        std::memcpy(kslot, ks, 256);
      std::memcpy(vslot, vs, 256);
      if (c->sink && t == 0) {  // the first token's fp16 row (reading R10)
        std::memcpy(cache->k_res + (unit * d.res_rows + d.ring) * 128, kslot, 256);
        std::memcpy(cache->v_res + (unit * d.res_rows + d.ring) * 128, vslot, 256);
      }
      if (Q_new > Q_old) {
        // Tokens [Q_old, Q_old + G) leave the window: gather them from the ring and quantize.
        std::vector<uint16_t> kt(static_cast<size_t>(G) * 128), vt(static_cast<size_t>(G) * 128);
        for (int i = 0; i < G; ++i) {
          const int64_t s = (Q_old + i) % d.ring;
          std::memcpy(&kt[i * 128], cache->k_res + (unit * d.res_rows + s) * 128, 256);
          std::memcpy(&vt[i * 128], cache->v_res + (unit * d.res_rows + s) * 128, 256);
        }
        quantize_span(c, cache, unit, Q_old, kt.data(), 128, vt.data(), 128);
      }
    }
    cache->seq_len[b] = t + 1;
  }
  return REF_OK;
}

// Dequantized key / value of token t (fp64, reading R6) or the FP16 residual copy.
static void key_row(const kvq_ref_config* c, const kvq_ref_cache* cache, int64_t unit, int64_t t, int64_t Q, double* out) {
  const Dims d = dims(c);
  if (t >= Q || (c->sink && t == 0)) {
    const int64_t row = (c->sink && t == 0) ? d.ring : t % d.ring;
    const uint16_t* r = cache->k_res + (unit * d.res_rows + row) * 128;
    for (int ch = 0; ch < 128; ++ch) out[ch] = half_to_float(r[ch]);
    return;
  }
  int64_t slot, ts;  // where token t is stored (reading R13)
  locate(c, cache, unit, t, &slot, &ts);
  const uint32_t* kbuf = cache->k_codes + slot * d.kwords;
  const int64_t g = ts / c->group_size;
  for (int ch = 0; ch < 128; ++ch) {
    int64_t word;
    int bit;
    key_pos(c, ts, ch, &word, &bit);
    const uint32_t code = (kbuf[word] >> bit) & ((1u << c->key_bits) - 1u);
    const int pos = key_param_index(c, ch);
    const double s = half_to_float(cache->k_scale[(slot * d.groups + g) * 128 + pos]);
    const double z = half_to_float(cache->k_zero[(slot * d.groups + g) * 128 + pos]);
    out[ch] = static_cast<double>(code) * s + z;
  }
  if (c->outliers) {  // the token's fp16 outlier replaces its entry (reading R12)
    const uint16_t ch = cache->k_out_ch[slot * d.slot_tokens + ts];
    if (ch < 128) out[ch] = half_to_float(cache->k_out_val[slot * d.slot_tokens + ts]);
  }
}

static void value_row(const kvq_ref_config* c, const kvq_ref_cache* cache, int64_t unit, int64_t t, int64_t Q, double* out) {
  const Dims d = dims(c);
  if (t >= Q || (c->sink && t == 0)) {
    const int64_t row = (c->sink && t == 0) ? d.ring : t % d.ring;
    const uint16_t* r = cache->v_res + (unit * d.res_rows + row) * 128;
    for (int ch = 0; ch < 128; ++ch) out[ch] = half_to_float(r[ch]);
    return;
  }
  int64_t slot, ts;  // where token t is stored (reading R13)
  locate(c, cache, unit, t, &slot, &ts);
  const uint32_t* vbuf = cache->v_codes + slot * d.vwords;
  for (int ch = 0; ch < 128; ++ch) {
    int64_t word;
    int bit;
    value_pos(c, ts, ch, &word, &bit);
    const uint32_t code = (vbuf[word] >> bit) & ((1u << c->value_bits) - 1u);
    const int j = ch / c->group_size;
    const double s = half_to_float(cache->v_scale[(slot * d.slot_tokens + ts) * d.vpt + j]);
    const double z = half_to_float(cache->v_zero[(slot * d.slot_tokens + ts) * d.vpt + j]);
    out[ch] = static_cast<double>(code) * s + z;
  }
  if (c->outliers) {  // the token's fp16 outlier replaces its entry (reading R12)
    const uint16_t ch = cache->v_out_ch[slot * d.slot_tokens + ts];
    if (ch < 128) out[ch] = half_to_float(cache->v_out_val[slot * d.slot_tokens + ts]);
  }
}

// RoPE of one key at position t (reading R11): channel pairs (i, i + 64) rotated by t * omega[i].
static void rope_rotate(double* k, int64_t t, const double* omega) {
  for (int i = 0; i < 64; ++i) {
    const double ang = static_cast<double>(t) * omega[i];
    const double cs = std::cos(ang), sn = std::sin(ang);
    const double a = k[i], b = k[i + 64];
    k[i] = a * cs - b * sn;
    k[i + 64] = a * sn + b * cs;
  }
}

// Exact attention of query head h of sequence b over the dequantized cache (reading R7).
static void decode_head(const kvq_ref_config* c, const kvq_ref_cache* cache, const uint16_t* q, double sm_scale,
                        int64_t b, int64_t h, double* out) {
  const int64_t gq = c->num_q_heads / c->num_kv_heads;
  const int64_t kvh = h / gq;
  const int64_t unit = b * c->num_kv_heads + kvh;
  const int64_t T = cache->seq_len[b];
  const int64_t Q = quantized_len(T, c->residual, c->group_size);
  double qv[128];
  const uint16_t* qs = q + (b * c->num_q_heads + h) * 128;
  for (int i = 0; i < 128; ++i) qv[i] = half_to_float(qs[i]);
  if (c->hadamard) wht128_f64(qv);
  std::vector<double> s(static_cast<size_t>(T));
  double row[128];
  double omega[64];  // RoPE frequencies theta^(-i/64)
  const bool rope = c->rope_theta > 0.0f;
  for (int i = 0; i < 64; ++i) omega[i] = rope ? std::pow(static_cast<double>(c->rope_theta), -i / 64.0) : 0.0;
  double mx = -INFINITY;
  for (int64_t t = 0; t < T; ++t) {
    key_row(c, cache, unit, t, Q, row);
    if (rope) rope_rotate(row, t, omega);
    double acc = 0.0;
    for (int i = 0; i < 128; ++i) acc += qv[i] * row[i];
    s[t] = sm_scale * acc;
    mx = std::max(mx, s[t]);
  }
  double o[128] = {0};
  double l = 0.0;
  for (int64_t t = 0; t < T; ++t) {
    const double p = std::exp(s[t] - mx);
    l += p;
    value_row(c, cache, unit, t, Q, row);
    for (int i = 0; i < 128; ++i) o[i] += p * row[i];
  }
  for (int i = 0; i < 128; ++i) out[i] = T > 0 ? o[i] / l : 0.0;
}

// Decode attention for every (sequence, query head). q: fp16 [B][Hq][128]; out: fp64 [B][Hq][128].
int kvq_ref_decode(const kvq_ref_config* c, const kvq_ref_cache* cache, const uint16_t* q, double sm_scale,
                   double* out, int nthreads) {
  int rc = check_config(c);
  if (rc) return rc;
  for (int64_t u = 0; u < static_cast<int64_t>(c->batch) * c->num_kv_heads; ++u)
    if (!pages_valid(c, cache, u, quantized_len(cache->seq_len[u / c->num_kv_heads], c->residual, c->group_size)))
      return REF_ERR_ARG;
  const int64_t rows = static_cast<int64_t>(c->batch) * c->num_q_heads;
  auto work = [&](int64_t r0, int64_t step) {
    for (int64_t r = r0; r < rows; r += step)
      decode_head(c, cache, q, sm_scale, r / c->num_q_heads, r % c->num_q_heads, out + r * 128);
  };
  if (nthreads <= 1) {
    work(0, 1);
  } else {
    std::vector<std::thread> pool;
    for (int i = 0; i < nthreads; ++i) pool.emplace_back(work, i, nthreads);
    for (auto& t : pool) t.join();
  }
  return REF_OK;
}

// ---- single-step helpers exposed for the oracle's own pins --------------------------------------
void kvq_ref_f16_to_f32(const uint16_t* in, float* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = half_to_float(in[i]);
}
void kvq_ref_f32_to_f16(const float* in, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = float_to_half(in[i]);
}
void kvq_ref_wht128_f32(float* x) { wht128_f32(x); }
void kvq_ref_wht128_f64(double* x) { wht128_f64(x); }
void kvq_ref_quantize_group(const uint16_t* x, int n, int bits, uint8_t* codes, uint16_t* scale, uint16_t* zero) {
  GroupQ g = quantize_group(x, n, 1, bits, codes, 1);
  *scale = g.scale;
  *zero = g.zero;
}
void kvq_ref_key_word_bit(int i, int c, int bits, int* word, int* bit) { key_word_bit(i, c, bits, word, bit); }
void kvq_ref_value_word_bit(int i, int c, int bits, int* word, int* bit) { value_word_bit(i, c, bits, word, bit); }
int kvq_ref_key_param_pos(int c) { return key_param_pos(c); }
void kvq_ref_key_word_bit_v2(int64_t t, int c, int bits, int64_t* word, int* bit) { key_word_bit_v2(t, c, bits, word, bit); }
void kvq_ref_value_word_bit_v2(int64_t t, int c, int bits, int64_t* word, int* bit) { value_word_bit_v2(t, c, bits, word, bit); }
int64_t kvq_ref_quantized_len(int64_t T, int R, int G) { return quantized_len(T, R, G); }

// Exhaustive check of the binary32 -> binary16 converter against the compiler's _Float16 conversion
// (round to nearest even) over every bit pattern in [lo, hi). Returns the number of mismatches
// (NaNs compare as "both NaN").
int64_t kvq_ref_check_f32_to_f16_range(uint64_t lo, uint64_t hi) {
  int64_t bad = 0;
  for (uint64_t u = lo; u < hi; ++u) {
    const uint32_t bits = static_cast<uint32_t>(u);
    float f;
    std::memcpy(&f, &bits, 4);
    const uint16_t mine = float_to_half(f);
    const _Float16 ref = static_cast<_Float16>(f);
    uint16_t rb;
    std::memcpy(&rb, &ref, 2);
    const bool mine_nan = (mine & 0x7c00u) == 0x7c00u && (mine & 0x3ffu);
    const bool ref_nan = (rb & 0x7c00u) == 0x7c00u && (rb & 0x3ffu);
    if (mine_nan || ref_nan) {
      bad += (mine_nan != ref_nan);
    } else {
      bad += (mine != rb);
    }
  }
  return bad;
}

}  // extern "C"
