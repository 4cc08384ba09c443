// Host-side NVFP4 packer for D_g and C_l (the export step of the DictLLM
// technical review's Algorithm 2: dictionary, per-layer codes, scales, support).
//
// Encoders are written from the OCP E2M1 / E4M3 definitions with plain IEEE
// fp32 arithmetic (compiled with -ffp-contract=off): E4M3 by scaling to the
// format's quantum and rounding half-to-even with nearbyintf, E2M1 by rounding
// on the three uniform sub-grids of its value set. Layouts are described in
// include/dictproj.h.
#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include "dictproj_internal.h"

namespace dictproj {

static inline float e4m3_decode(uint8_t c) {
  const int e = (c >> 3) & 15, m = c & 7;
  const float mag = e == 0 ? std::ldexp((float)m, -9) : std::ldexp(1.0f + (float)m / 8.0f, e - 7);
  return (c & 0x80) ? -mag : mag;
}

// Nearest E4M3 code to r >= 0 (finite), ties to even, saturating at 448 (0x7E).
static inline uint8_t e4m3_encode_nonneg(float r) {
  if (!(r > 0.0f)) return 0;
  if (r >= 448.0f) return 0x7E;
  int e2;
  std::frexp(r, &e2);        // r = f * 2^e2, f in [0.5, 1)  ->  floor(log2 r) = e2 - 1
  int E = e2 - 1;
  if (E < -6) E = -6;        // subnormal range shares the 2^-6 binade's quantum
  const float n = std::nearbyintf(std::ldexp(r, 3 - E));  // quanta of 2^(E-3), half-to-even
  int ni = (int)n;
  if (E == -6 && ni < 8) return (uint8_t)ni;  // subnormal (or zero)
  if (ni == 16) { ni = 8; E += 1; }           // rounded up into the next binade
  if (E > 8 || (E == 8 && ni > 14)) return 0x7E;
  return (uint8_t)(((E + 7) << 3) | (ni - 8));
}

// Nearest E2M1 code to q, ties to even mantissa, saturating at 6; -0 -> 0.
static inline uint8_t e2m1_encode(float q) {
  const float a = std::fabs(q);
  uint8_t mag;
  if (a >= 6.0f) {
    mag = 7;
  } else if (a < 2.0f) {            // grid 0, .5, 1, 1.5, 2  -> codes 0..4
    mag = (uint8_t)std::nearbyintf(a * 2.0f);
  } else if (a < 4.0f) {            // grid 2, 3, 4           -> codes 4..6
    mag = (uint8_t)((int)std::nearbyintf(a) + 2);
  } else {                          // grid 4, 6              -> codes 6, 7
    mag = (uint8_t)((int)std::nearbyintf(a * 0.5f) + 4);
  }
  return (q < 0.0f && mag != 0) ? (uint8_t)(mag | 8) : mag;
}

// IEEE binary16 bits of x, round to nearest even, written from the format's
// definition: quanta of 2^(E-10) in the binade [2^E, 2^(E+1)), 2^-24 below 2^-14
// (subnormals; a value that rounds up to 2^-14 lands on the first normal code).
// Returns false if |x| rounds beyond the largest finite value (65504).
static inline bool fp16_encode(float x, uint16_t* out) {
  const float a = std::fabs(x);
  const uint16_t sign = std::signbit(x) ? 0x8000 : 0;
  uint32_t bits;
  if (a < 0x1p-14f) {
    bits = (uint32_t)std::nearbyintf(std::ldexp(a, 24));  // 0 .. 1024
  } else {
    int e2;
    std::frexp(a, &e2);
    int E = e2 - 1;
    uint32_t n = (uint32_t)std::nearbyintf(std::ldexp(a, 10 - E));  // 1024 .. 2048
    if (n == 2048) {
      n = 1024;
      E += 1;
    }
    if (E > 15) return false;
    bits = ((uint32_t)(E + 15) << 10) | (n - 1024);
  }
  *out = (uint16_t)(sign | bits);
  return true;
}

static inline float tensor_scale_from_amax(float amax) {
  if (amax == 0.0f) return 1.0f;
  return amax / 2688.0f;
}

// Quantise one block of 16 values given the tensor scale; writes 16 codes and
// returns the scale code.
static inline uint8_t quantize_block(const float* x, float s_t, uint8_t* codes16) {
  float amax_b = 0.0f;
  for (int i = 0; i < 16; ++i) amax_b = std::fmax(amax_b, std::fabs(x[i]));
  const float den = 6.0f * s_t;
  const float r = amax_b / den;
  const uint8_t sc = e4m3_encode_nonneg(r);
  const float scale = e4m3_decode(sc) * s_t;
  for (int i = 0; i < 16; ++i) codes16[i] = scale == 0.0f ? 0 : e2m1_encode(x[i] / scale);
  return sc;
}

template <class F>
static void parallel_for(size_t n, F&& f) {
  unsigned nt = std::thread::hardware_concurrency();
  if (nt == 0) nt = 1;
  if (nt > 32) nt = 32;
  if (n < 4096 || nt == 1) { f(size_t(0), n); return; }
  std::vector<std::thread> th;
  const size_t chunk = (n + nt - 1) / nt;
  for (unsigned t = 0; t < nt; ++t) {
    const size_t a = t * chunk, b = std::min(n, a + chunk);
    if (a >= b) break;
    th.emplace_back([&, a, b] {
      std::fesetround(FE_TONEAREST);
      f(a, b);
    });
  }
  for (auto& t : th) t.join();
}

int pack_group_host(const float* D, int d_in, int k, uint8_t* codes, uint8_t* scales, float* s_D) {
  if (!D || !codes || !scales || !s_D) return fail(DICTPROJ_ERR_NULL, "pack_group_host: NULL pointer");
  if (d_in <= 0 || k <= 0 || d_in % 16) return fail(DICTPROJ_ERR_SHAPE, "pack_group_host: need d_in > 0, d_in %% 16 == 0, k > 0 (got d_in=%d k=%d)", d_in, k);
  std::fesetround(FE_TONEAREST);
  const size_t n = (size_t)d_in * k;
  // amax and finiteness
  std::vector<float> part(64, 0.0f);
  std::vector<int> bad(64, 0);
  {
    unsigned nt = std::min<unsigned>(64, std::max(1u, std::thread::hardware_concurrency()));
    std::vector<std::thread> th;
    const size_t chunk = (n + nt - 1) / nt;
    for (unsigned t = 0; t < nt; ++t) {
      th.emplace_back([&, t] {
        const size_t a = t * chunk, b = std::min(n, a + chunk);
        float m = 0.0f;
        for (size_t i = a; i < b; ++i) {
          if (!std::isfinite(D[i])) { bad[t] = 1; break; }
          m = std::fmax(m, std::fabs(D[i]));
        }
        part[t] = m;
      });
    }
    for (auto& t : th) t.join();
  }
  float amax = 0.0f;
  for (int t = 0; t < 64; ++t) {
    if (bad[t]) return fail(DICTPROJ_ERR_VALUE, "pack_group_host: non-finite value in D");
    amax = std::fmax(amax, part[t]);
  }
  const float s = tensor_scale_from_amax(amax);
  const int nb = d_in / 16;
  // one task per atom: gather its d_in column of D (row-major d_in x k) into blocks
  parallel_for((size_t)k, [&](size_t a0, size_t a1) {
    float blk[16];
    uint8_t c16[16];
    for (size_t j = a0; j < a1; ++j) {
      uint8_t* crow = codes + j * (size_t)(d_in / 2);
      uint8_t* srow = scales + j * (size_t)nb;
      for (int b = 0; b < nb; ++b) {
        for (int i = 0; i < 16; ++i) blk[i] = D[(size_t)(16 * b + i) * k + j];
        srow[b] = quantize_block(blk, s, c16);
        for (int i = 0; i < 8; ++i) crow[8 * b + i] = (uint8_t)(c16[2 * i] | (c16[2 * i + 1] << 4));
      }
    }
  });
  *s_D = s;
  return DICTPROJ_OK;
}

int layer_packed_entries(const int32_t* col_ptr, int k, int d_out, size_t* total) {
  if (!col_ptr || !total) return fail(DICTPROJ_ERR_NULL, "layer_packed_entries: NULL pointer");
  if (k <= 0 || k > 65535 || d_out <= 0) return fail(DICTPROJ_ERR_SHAPE, "layer: need 0 < k <= 65535 and d_out > 0 (got k=%d d_out=%d)", k, d_out);
  if (col_ptr[0] != 0) return fail(DICTPROJ_ERR_RANGE, "layer: col_ptr[0] must be 0");
  size_t t = 0;
  for (int o = 0; o < d_out; ++o) {
    const int64_t n = (int64_t)col_ptr[o + 1] - col_ptr[o];
    if (n < 0 || n > k) return fail(DICTPROJ_ERR_RANGE, "layer: column %d has %lld entries (k=%d)", o, (long long)n, k);
    t += (size_t)((n + 15) / 16) * 16;
  }
  *total = t;
  return DICTPROJ_OK;
}

// Quantise C_l and lay it out; the support goes to idx + seg_start (u8 index,
// Eq. (12) a = 8) when they are given and to a bitmap (Eq. (12) a = 0, h = 1)
// when `bitmap` is given. Codes, scales and padding are the same either way.
static int pack_layer_core(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k,
                           int d_out, uint32_t* pcol_ptr, uint32_t* nnz, uint8_t* codes, uint8_t* scales,
                           uint8_t* idx, uint16_t* seg_start, uint32_t* bitmap, float* s_C) {
  size_t total = 0;
  int st = layer_packed_entries(col_ptr, k, d_out, &total);
  if (st) return st;
  const size_t nz = (size_t)col_ptr[d_out];
  if (nz && (!atom_idx || !vals)) return fail(DICTPROJ_ERR_NULL, "pack_layer_host: NULL atom_idx/vals");
  std::fesetround(FE_TONEAREST);
  float amax = 0.0f;
  for (size_t i = 0; i < nz; ++i) {
    if (!std::isfinite(vals[i])) return fail(DICTPROJ_ERR_VALUE, "pack_layer_host: non-finite value at %zu", i);
    amax = std::fmax(amax, std::fabs(vals[i]));
  }
  for (int o = 0; o < d_out; ++o) {
    for (int32_t q = col_ptr[o]; q < col_ptr[o + 1]; ++q) {
      const int32_t a = atom_idx[q];
      if (a < 0 || a >= k) return fail(DICTPROJ_ERR_RANGE, "pack_layer_host: atom %d out of [0,%d) in column %d", a, k, o);
      if (q > col_ptr[o] && a <= atom_idx[q - 1]) return fail(DICTPROJ_ERR_RANGE, "pack_layer_host: atoms not ascending/unique in column %d", o);
    }
  }
  const float s = tensor_scale_from_amax(amax);
  const int nseg = (k + 255) / 256;
  pcol_ptr[0] = 0;
  for (int o = 0; o < d_out; ++o) {
    const uint32_t n = (uint32_t)(col_ptr[o + 1] - col_ptr[o]);
    nnz[o] = n;
    pcol_ptr[o + 1] = pcol_ptr[o] + ((n + 15) / 16) * 16;
  }
  parallel_for((size_t)d_out, [&](size_t o0, size_t o1) {
    float blk[16];
    uint8_t c16[16];
    for (size_t o = o0; o < o1; ++o) {
      const int32_t b0 = col_ptr[o];
      const int32_t n = col_ptr[o + 1] - b0;
      const uint32_t p0 = pcol_ptr[o];
      const uint32_t P = pcol_ptr[o + 1] - p0;
      if (seg_start) {  // segment starts: entries are ascending, so one pass
        int q = 0;
        for (int sgi = 0; sgi < nseg; ++sgi) {
          while (q < n && atom_idx[b0 + q] < 256 * sgi) ++q;
          seg_start[o * (size_t)nseg + sgi] = (uint16_t)q;
        }
      }
      if (bitmap) {
        const int words = (k + 31) / 32;
        uint32_t* row = bitmap + o * (size_t)words;
        for (int w = 0; w < words; ++w) row[w] = 0u;
        for (int q = 0; q < n; ++q) row[atom_idx[b0 + q] >> 5] |= 1u << (atom_idx[b0 + q] & 31);
      }
      for (uint32_t e = 0; e < P; e += 16) {
        for (int i = 0; i < 16; ++i) {
          const uint32_t qq = e + i;
          blk[i] = qq < (uint32_t)n ? vals[b0 + qq] : 0.0f;
          if (idx) idx[p0 + qq] = qq < (uint32_t)n ? (uint8_t)(atom_idx[b0 + qq] & 255) : 0;
        }
        scales[(p0 + e) / 16] = quantize_block(blk, s, c16);
        for (int i = 0; i < 8; ++i) codes[(p0 + e) / 2 + i] = (uint8_t)(c16[2 * i] | (c16[2 * i + 1] << 4));
      }
    }
  });
  *s_C = s;
  return DICTPROJ_OK;
}

int pack_layer_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k,
                    int d_out, uint32_t* pcol_ptr, uint32_t* nnz, uint8_t* codes, uint8_t* scales,
                    uint8_t* idx, uint16_t* seg_start, float* s_C) {
  if (!col_ptr || !pcol_ptr || !nnz || !codes || !scales || !idx || !seg_start || !s_C)
    return fail(DICTPROJ_ERR_NULL, "pack_layer_host: NULL pointer");
  return pack_layer_core(col_ptr, atom_idx, vals, k, d_out, pcol_ptr, nnz, codes, scales, idx, seg_start, nullptr,
                         s_C);
}

// C_l with its stored values in one of Table 4's coefficient formats (FP16,
// FP8 E4M3, INT8) and the u8 index of the NVFP4 layout: one code per stored
// entry (padding entries 0), one fp32 per-tensor scale (1 for FP16).
int pack_layer_fmt_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k, int d_out,
                        int fmt, uint32_t* pcol_ptr, uint32_t* nnz, void* values, uint8_t* idx,
                        uint16_t* seg_start, float* s_C) {
  if (fmt == DICTPROJ_CFMT_NVFP4)
    return fail(DICTPROJ_ERR_RANGE, "pack_layer_fmt_host: NVFP4 coefficients are packed by dictproj_pack_layer_host");
  if (fmt != DICTPROJ_CFMT_FP16 && fmt != DICTPROJ_CFMT_FP8 && fmt != DICTPROJ_CFMT_INT8)
    return fail(DICTPROJ_ERR_RANGE, "pack_layer_fmt_host: unknown coefficient format %d", fmt);
  if (!col_ptr || !pcol_ptr || !nnz || !values || !idx || !seg_start || !s_C)
    return fail(DICTPROJ_ERR_NULL, "pack_layer_fmt_host: NULL pointer");
  size_t total = 0;
  int st = layer_packed_entries(col_ptr, k, d_out, &total);
  if (st) return st;
  // the index, padding and column pointers of the NVFP4 layout (its codes and scales are discarded)
  std::vector<uint8_t> codes(total / 2 + 1), scales(total / 16 + 1);
  float s_nv = 0.f;
  if ((st = pack_layer_core(col_ptr, atom_idx, vals, k, d_out, pcol_ptr, nnz, codes.data(), scales.data(), idx,
                            seg_start, nullptr, &s_nv)))
    return st;
  const size_t nz = (size_t)col_ptr[d_out];
  float amax = 0.0f;
  for (size_t i = 0; i < nz; ++i) amax = std::fmax(amax, std::fabs(vals[i]));
  float s = 1.0f;
  if (fmt == DICTPROJ_CFMT_FP8) s = amax == 0.0f ? 1.0f : amax / 448.0f;
  if (fmt == DICTPROJ_CFMT_INT8) s = amax == 0.0f ? 1.0f : amax / 127.0f;
  std::fesetround(FE_TONEAREST);
  for (int o = 0; o < d_out; ++o) {
    const int32_t b0 = col_ptr[o], n = col_ptr[o + 1] - b0;
    const uint32_t p0 = pcol_ptr[o], P = pcol_ptr[o + 1] - p0;
    for (uint32_t q = 0; q < P; ++q) {
      const float x = q < (uint32_t)n ? vals[b0 + q] : 0.0f;
      if (fmt == DICTPROJ_CFMT_FP16) {
        uint16_t h;
        if (!fp16_encode(x, &h))
          return fail(DICTPROJ_ERR_VALUE, "pack_layer_fmt_host: value %g of column %d outside the fp16 range", x, o);
        static_cast<uint16_t*>(values)[p0 + q] = h;
      } else if (fmt == DICTPROJ_CFMT_FP8) {
        const float r = x / s;
        const uint8_t mag = e4m3_encode_nonneg(std::fabs(r));
        static_cast<uint8_t*>(values)[p0 + q] = (r < 0.0f && mag) ? (uint8_t)(mag | 0x80) : mag;
      } else {
        float c = std::nearbyintf(x / s);
        c = std::fmin(127.0f, std::fmax(-127.0f, c));
        static_cast<int8_t*>(values)[p0 + q] = (int8_t)c;
      }
    }
  }
  *s_C = s;
  return DICTPROJ_OK;
}

// C_l with block-structured support: every column's atoms are whole aligned
// blocks of 16; a kept block is one NVFP4 block (codes, scale) with a uint16
// block number. blk_ptr counts kept blocks before each column.
int pack_layer_blocks_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k, int d_out,
                           uint32_t* blk_ptr, uint16_t* blk_idx, uint8_t* codes, uint8_t* scales, float* s_C) {
  if (!col_ptr || !blk_ptr || !blk_idx || !codes || !scales || !s_C)
    return fail(DICTPROJ_ERR_NULL, "pack_layer_blocks_host: NULL pointer");
  if (k <= 0 || k % 16 || k > 65535 || d_out <= 0)
    return fail(DICTPROJ_ERR_SHAPE, "pack_layer_blocks_host: need 0 < k <= 65535, k %% 16 == 0, d_out > 0");
  if (col_ptr[0] != 0) return fail(DICTPROJ_ERR_RANGE, "pack_layer_blocks_host: col_ptr[0] must be 0");
  for (int o = 0; o < d_out; ++o) {
    const int32_t b0 = col_ptr[o], n = col_ptr[o + 1] - b0;
    if (n < 0 || n > k || n % 16)
      return fail(DICTPROJ_ERR_RANGE, "pack_layer_blocks_host: column %d holds %d entries, not whole 16-atom blocks", o,
                  n);
    for (int32_t q = 0; q < n; ++q)
      if (atom_idx[b0 + q] != (atom_idx[b0 + (q & ~15)] & ~15) + (q & 15) || (atom_idx[b0 + (q & ~15)] & 15))
        return fail(DICTPROJ_ERR_RANGE, "pack_layer_blocks_host: column %d is not a union of aligned 16-atom blocks", o);
  }
  // values, padding-free blocks and scales exactly as the u8 layout packs them
  size_t total = 0;
  int st = layer_packed_entries(col_ptr, k, d_out, &total);
  if (st) return st;
  std::vector<uint32_t> pptr(d_out + 1), nnz(d_out);
  std::vector<uint8_t> idx(total + 1);
  std::vector<uint16_t> ss((size_t)d_out * ((k + 255) / 256));
  if ((st = pack_layer_core(col_ptr, atom_idx, vals, k, d_out, pptr.data(), nnz.data(), codes, scales, idx.data(),
                            ss.data(), nullptr, s_C)))
    return st;
  blk_ptr[0] = 0;
  for (int o = 0; o < d_out; ++o) {
    const int32_t b0 = col_ptr[o], nb = (col_ptr[o + 1] - b0) / 16;
    for (int32_t b = 0; b < nb; ++b) blk_idx[blk_ptr[o] + b] = (uint16_t)(atom_idx[b0 + 16 * b] >> 4);
    blk_ptr[o + 1] = blk_ptr[o] + (uint32_t)nb;
  }
  return DICTPROJ_OK;
}

int pack_layer_bitmap_host(const int32_t* col_ptr, const int32_t* atom_idx, const float* vals, int k, int d_out,
                           uint32_t* pcol_ptr, uint32_t* nnz, uint8_t* codes, uint8_t* scales, uint32_t* bitmap,
                           float* s_C) {
  if (!col_ptr || !pcol_ptr || !nnz || !codes || !scales || !bitmap || !s_C)
    return fail(DICTPROJ_ERR_NULL, "pack_layer_bitmap_host: NULL pointer");
  return pack_layer_core(col_ptr, atom_idx, vals, k, d_out, pcol_ptr, nnz, codes, scales, nullptr, nullptr, bitmap,
                         s_C);
}

}  // namespace dictproj
