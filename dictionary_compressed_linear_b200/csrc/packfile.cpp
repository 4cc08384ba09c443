// Host-side helpers around the packed factors (no device code):
//
// * the rank budget of Eq. (3) and the value counts of Eq. (2) of the DictLLM
//   technical review ("The budget: trading shared rank against sparsity");
// * the export step of the review's Algorithm 2 (step 10: export the
//   dictionary, per-layer codes, scales and support) as a file format: the
//   packed byte arrays of one group or one layer, behind a small header with
//   the shapes, the fp32 tensor scale and a 64-bit FNV-1a checksum of the
//   payload. All fields are little-endian.
//
//   header (64 bytes):
//     char     magic[8]   "DPJGRP1\0" (group) or "DPJLYR1\0" (layer)
//     uint32   a, b       group: d_in, k            layer: k, d_out
//     uint32   c          group: 0                  layer: nseg = ceil(k / 256)
//     float    s          s_D or s_C
//     uint64   total      group: 0                  layer: padded entries
//     uint64   payload    bytes after the header
//     uint64   checksum   FNV-1a 64 of the payload
//     uint8    reserved[16] = 0
//   payload, group: codes [k][d_in/2], scales [k][d_in/16]
//   payload, layer: col_ptr u32[d_out+1], codes [total/2], scales [total/16],
//                   idx [total], seg_start u16[d_out][nseg]
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <vector>

#include "dictproj.h"
#include "dictproj_internal.h"

namespace dictproj {
namespace {

constexpr char kGroupMagic[8] = {'D', 'P', 'J', 'G', 'R', 'P', '1', 0};
constexpr char kLayerMagic[8] = {'D', 'P', 'J', 'L', 'Y', 'R', '1', 0};

struct FileHeader {
  char magic[8];
  uint32_t a, b, c;
  float s;
  uint64_t total, payload, checksum;
  uint8_t reserved[16];
};
static_assert(sizeof(FileHeader) == 64, "header layout");

struct Fnv {
  uint64_t h = 1469598103934665603ull;
  void add(const void* p, size_t n) {
    const uint8_t* b = static_cast<const uint8_t*>(p);
    for (size_t i = 0; i < n; ++i) {
      h ^= b[i];
      h *= 1099511628211ull;
    }
  }
};

struct Part {
  const void* p;
  size_t n;
};

int write_file(const char* path, FileHeader h, const std::vector<Part>& parts, const char* what) {
  Fnv f;
  uint64_t payload = 0;
  for (const Part& x : parts) {
    f.add(x.p, x.n);
    payload += x.n;
  }
  h.payload = payload;
  h.checksum = f.h;
  FILE* fp = std::fopen(path, "wb");
  if (!fp) return fail(DICTPROJ_ERR_IO, "%s: cannot open '%s' for writing", what, path);
  bool ok = std::fwrite(&h, sizeof h, 1, fp) == 1;
  for (const Part& x : parts)
    if (ok && x.n) ok = std::fwrite(x.p, 1, x.n, fp) == x.n;
  ok = (std::fclose(fp) == 0) && ok;
  if (!ok) return fail(DICTPROJ_ERR_IO, "%s: write to '%s' failed", what, path);
  return DICTPROJ_OK;
}

int read_header(const char* path, const char* magic, FileHeader* h, const char* what) {
  FILE* fp = std::fopen(path, "rb");
  if (!fp) return fail(DICTPROJ_ERR_IO, "%s: cannot open '%s'", what, path);
  const bool ok = std::fread(h, sizeof *h, 1, fp) == 1;
  std::fclose(fp);
  if (!ok) return fail(DICTPROJ_ERR_VALUE, "%s: '%s' is shorter than a header", what, path);
  if (std::memcmp(h->magic, magic, 8) != 0) return fail(DICTPROJ_ERR_VALUE, "%s: '%s' has the wrong magic", what, path);
  return DICTPROJ_OK;
}

// Read the payload into the parts (sizes already checked against the header),
// then verify the file ends there and the checksum matches.
int read_payload(const char* path, const FileHeader& h, const std::vector<std::pair<void*, size_t>>& parts,
                 const char* what) {
  FILE* fp = std::fopen(path, "rb");
  if (!fp) return fail(DICTPROJ_ERR_IO, "%s: cannot open '%s'", what, path);
  bool ok = std::fseek(fp, (long)sizeof(FileHeader), SEEK_SET) == 0;
  Fnv f;
  for (const auto& x : parts) {
    if (ok && x.second) ok = std::fread(x.first, 1, x.second, fp) == x.second;
    if (ok) f.add(x.first, x.second);
  }
  const bool at_end = ok && std::fgetc(fp) == EOF;
  std::fclose(fp);
  if (!ok) return fail(DICTPROJ_ERR_VALUE, "%s: '%s' is truncated", what, path);
  if (!at_end) return fail(DICTPROJ_ERR_VALUE, "%s: '%s' has trailing bytes", what, path);
  if (f.h != h.checksum) return fail(DICTPROJ_ERR_VALUE, "%s: checksum mismatch in '%s'", what, path);
  return DICTPROJ_OK;
}

int nseg_of(int k) { return (k + 255) / 256; }

}  // namespace
}  // namespace dictproj

using namespace dictproj;

extern "C" {

int dictproj_rank_for_budget(double rho_fac, int n, int d_in, int d_out, int align, int* k_out) {
  clear_error();
  if (!k_out) return fail(DICTPROJ_ERR_NULL, "rank_for_budget: NULL output");
  if (!(rho_fac >= 0.0 && rho_fac < 1.0)) return fail(DICTPROJ_ERR_RANGE, "rank_for_budget: need 0 <= rho_fac < 1");
  if (n < 1 || d_in < 1 || d_out < 1 || align < 1)
    return fail(DICTPROJ_ERR_SHAPE, "rank_for_budget: need n, d_in, d_out, align >= 1");
  const double k = (1.0 - rho_fac) * (double)n * (double)d_in * (double)d_out / ((double)d_in + (double)n * d_out);
  const long long kf = (long long)std::floor(k);
  const long long ka = kf / align * align;  // round down: the value budget binds
  if (ka < 1) return fail(DICTPROJ_ERR_RANGE, "rank_for_budget: the budget leaves no rank (k = %.3f, align %d)", k, align);
  if (ka > 2147483647ll) return fail(DICTPROJ_ERR_RANGE, "rank_for_budget: rank overflows int");
  *k_out = (int)ka;
  return DICTPROJ_OK;
}

int dictproj_budget(int n, int d_in, int d_out, int k, double p, double* N0, double* Np, double* rho, double* G) {
  clear_error();
  if (n < 1 || d_in < 1 || d_out < 1 || k < 1) return fail(DICTPROJ_ERR_SHAPE, "budget: need n, d_in, d_out, k >= 1");
  if (!(p >= 0.0 && p <= 1.0)) return fail(DICTPROJ_ERR_RANGE, "budget: need 0 <= p <= 1");
  const double n0 = (double)n * d_in * d_out;
  const double np = (double)d_in * k + (double)n * (1.0 - p) * k * d_out;
  if (N0) *N0 = n0;
  if (Np) *Np = np;
  if (rho) *rho = 1.0 - np / n0;
  if (G) *G = n0 / np;
  return DICTPROJ_OK;
}

int dictproj_group_file_write(const char* path, const uint8_t* codes, const uint8_t* scales, float s_D, int d_in,
                              int k) {
  clear_error();
  if (!path || !codes || !scales) return fail(DICTPROJ_ERR_NULL, "group_file_write: NULL pointer");
  if (d_in <= 0 || d_in % 32 || k <= 0 || k % 16 || k > 65535)
    return fail(DICTPROJ_ERR_SHAPE, "group_file_write: need d_in %% 32 == 0, 0 < k <= 65535, k %% 16 == 0");
  if (!(s_D > 0.0f) || !std::isfinite(s_D)) return fail(DICTPROJ_ERR_VALUE, "group_file_write: s_D must be finite and > 0");
  FileHeader h{};
  std::memcpy(h.magic, kGroupMagic, 8);
  h.a = (uint32_t)d_in;
  h.b = (uint32_t)k;
  h.s = s_D;
  const size_t nc = (size_t)d_in * k / 2, ns = (size_t)d_in * k / 16;
  return write_file(path, h, {{codes, nc}, {scales, ns}}, "group_file_write");
}

int dictproj_group_file_info(const char* path, int* d_in, int* k) {
  clear_error();
  if (!path) return fail(DICTPROJ_ERR_NULL, "group_file_info: NULL path");
  FileHeader h;
  int st = read_header(path, kGroupMagic, &h, "group_file_info");
  if (st) return st;
  if (d_in) *d_in = (int)h.a;
  if (k) *k = (int)h.b;
  return DICTPROJ_OK;
}

int dictproj_group_file_read(const char* path, uint8_t* codes, uint8_t* scales, float* s_D, int d_in, int k) {
  clear_error();
  if (!path || !codes || !scales || !s_D) return fail(DICTPROJ_ERR_NULL, "group_file_read: NULL pointer");
  FileHeader h;
  int st = read_header(path, kGroupMagic, &h, "group_file_read");
  if (st) return st;
  if ((int)h.a != d_in || (int)h.b != k)
    return fail(DICTPROJ_ERR_MISMATCH, "group_file_read: file holds d_in=%u k=%u, buffers are for d_in=%d k=%d", h.a,
                h.b, d_in, k);
  if (d_in <= 0 || d_in % 32 || k <= 0 || k % 16) return fail(DICTPROJ_ERR_VALUE, "group_file_read: bad shape in file");
  const size_t nc = (size_t)d_in * k / 2, ns = (size_t)d_in * k / 16;
  if (h.payload != nc + ns) return fail(DICTPROJ_ERR_VALUE, "group_file_read: payload size does not match the shape");
  if (!(h.s > 0.0f) || !std::isfinite(h.s)) return fail(DICTPROJ_ERR_VALUE, "group_file_read: bad s_D in file");
  if ((st = read_payload(path, h, {{codes, nc}, {scales, ns}}, "group_file_read"))) return st;
  *s_D = h.s;
  return DICTPROJ_OK;
}

int dictproj_layer_file_write(const char* path, const uint32_t* pcol_ptr, const uint8_t* codes, const uint8_t* scales,
                              const uint8_t* idx, const uint16_t* seg_start, float s_C, int k, int d_out) {
  clear_error();
  if (!path || !pcol_ptr || !codes || !scales || !idx || !seg_start)
    return fail(DICTPROJ_ERR_NULL, "layer_file_write: NULL pointer");
  if (k <= 0 || k % 16 || k > 65535 || d_out <= 0)
    return fail(DICTPROJ_ERR_SHAPE, "layer_file_write: need 0 < k <= 65535, k %% 16 == 0, d_out > 0");
  if (!(s_C > 0.0f) || !std::isfinite(s_C)) return fail(DICTPROJ_ERR_VALUE, "layer_file_write: s_C must be finite and > 0");
  if (pcol_ptr[0] != 0) return fail(DICTPROJ_ERR_RANGE, "layer_file_write: col_ptr[0] must be 0");
  for (int o = 0; o < d_out; ++o)
    if (pcol_ptr[o + 1] < pcol_ptr[o] || (pcol_ptr[o + 1] - pcol_ptr[o]) % 16)
      return fail(DICTPROJ_ERR_RANGE, "layer_file_write: column %d has a bad padded length", o);
  const size_t total = pcol_ptr[d_out];
  const int nseg = nseg_of(k);
  FileHeader h{};
  std::memcpy(h.magic, kLayerMagic, 8);
  h.a = (uint32_t)k;
  h.b = (uint32_t)d_out;
  h.c = (uint32_t)nseg;
  h.s = s_C;
  h.total = total;
  return write_file(path, h,
                    {{pcol_ptr, 4 * ((size_t)d_out + 1)},
                     {codes, total / 2},
                     {scales, total / 16},
                     {idx, total},
                     {seg_start, 2 * (size_t)d_out * nseg}},
                    "layer_file_write");
}

int dictproj_layer_file_info(const char* path, int* k, int* d_out, size_t* total) {
  clear_error();
  if (!path) return fail(DICTPROJ_ERR_NULL, "layer_file_info: NULL path");
  FileHeader h;
  int st = read_header(path, kLayerMagic, &h, "layer_file_info");
  if (st) return st;
  if (k) *k = (int)h.a;
  if (d_out) *d_out = (int)h.b;
  if (total) *total = (size_t)h.total;
  return DICTPROJ_OK;
}

int dictproj_layer_file_read(const char* path, uint32_t* pcol_ptr, uint8_t* codes, uint8_t* scales, uint8_t* idx,
                             uint16_t* seg_start, float* s_C, int k, int d_out, size_t total) {
  clear_error();
  if (!path || !pcol_ptr || !codes || !scales || !idx || !seg_start || !s_C)
    return fail(DICTPROJ_ERR_NULL, "layer_file_read: NULL pointer");
  FileHeader h;
  int st = read_header(path, kLayerMagic, &h, "layer_file_read");
  if (st) return st;
  if ((int)h.a != k || (int)h.b != d_out || h.total != (uint64_t)total)
    return fail(DICTPROJ_ERR_MISMATCH, "layer_file_read: file holds k=%u d_out=%u total=%llu, buffers differ", h.a, h.b,
                (unsigned long long)h.total);
  if (k <= 0 || k % 16 || d_out <= 0 || total % 16 || (int)h.c != nseg_of(k))
    return fail(DICTPROJ_ERR_VALUE, "layer_file_read: bad shape in file");
  const size_t sizes[5] = {4 * ((size_t)d_out + 1), total / 2, total / 16, total, 2 * (size_t)d_out * h.c};
  if (h.payload != sizes[0] + sizes[1] + sizes[2] + sizes[3] + sizes[4])
    return fail(DICTPROJ_ERR_VALUE, "layer_file_read: payload size does not match the shape");
  if (!(h.s > 0.0f) || !std::isfinite(h.s)) return fail(DICTPROJ_ERR_VALUE, "layer_file_read: bad s_C in file");
  if ((st = read_payload(path, h,
                         {{pcol_ptr, sizes[0]}, {codes, sizes[1]}, {scales, sizes[2]}, {idx, sizes[3]},
                          {seg_start, sizes[4]}},
                         "layer_file_read")))
    return st;
  if (pcol_ptr[0] != 0 || pcol_ptr[d_out] != total) return fail(DICTPROJ_ERR_VALUE, "layer_file_read: bad col_ptr in file");
  *s_C = h.s;
  return DICTPROJ_OK;
}

// ---- device handles <-> files: compositions of the calls above with the
// exports / uploads of the ABI (the device parts need a GPU).

int dictproj_group_save(const dictproj_group* g, const char* path) {
  clear_error();
  if (!g || !path) return fail(DICTPROJ_ERR_NULL, "group_save: NULL pointer");
  int d_in = 0, k = 0;
  int st = dictproj_group_info(g, &d_in, &k, nullptr);
  if (st) return st;
  std::vector<uint8_t> codes((size_t)d_in * k / 2), scales((size_t)d_in * k / 16);
  float s = 0.0f;
  if ((st = dictproj_group_export(g, codes.data(), scales.data(), &s))) return st;
  return dictproj_group_file_write(path, codes.data(), scales.data(), s, d_in, k);
}

int dictproj_group_load(const char* path, int max_tokens, dictproj_group** out) {
  clear_error();
  if (!path || !out) return fail(DICTPROJ_ERR_NULL, "group_load: NULL pointer");
  *out = nullptr;
  int d_in = 0, k = 0;
  int st = dictproj_group_file_info(path, &d_in, &k);
  if (st) return st;
  if (d_in <= 0 || d_in % 32 || k <= 0 || k % 16 || k > 65535) return fail(DICTPROJ_ERR_VALUE, "group_load: bad shape in file");
  std::vector<uint8_t> codes((size_t)d_in * k / 2), scales((size_t)d_in * k / 16);
  float s = 0.0f;
  if ((st = dictproj_group_file_read(path, codes.data(), scales.data(), &s, d_in, k))) return st;
  return dictproj_group_upload(codes.data(), scales.data(), s, d_in, k, max_tokens, out);
}

int dictproj_layer_save(const dictproj_layer* l, const char* path) {
  clear_error();
  if (!l || !path) return fail(DICTPROJ_ERR_NULL, "layer_save: NULL pointer");
  int k = 0, d_out = 0;
  size_t total = 0;
  int st = dictproj_layer_info(l, &k, &d_out, &total, nullptr);
  if (st) return st;
  const size_t nseg = (size_t)(k + 255) / 256;
  std::vector<uint32_t> col_ptr((size_t)d_out + 1);
  std::vector<uint8_t> codes(total / 2), scales(total / 16), idx(total);
  std::vector<uint16_t> ss((size_t)d_out * nseg);
  float s = 0.0f;
  if ((st = dictproj_layer_export(l, col_ptr.data(), codes.data(), scales.data(), idx.data(), ss.data(), &s))) return st;
  return dictproj_layer_file_write(path, col_ptr.data(), codes.data(), scales.data(), idx.data(), ss.data(), s, k, d_out);
}

int dictproj_layer_load(const char* path, dictproj_layer** out) {
  clear_error();
  if (!path || !out) return fail(DICTPROJ_ERR_NULL, "layer_load: NULL pointer");
  *out = nullptr;
  int k = 0, d_out = 0;
  size_t total = 0;
  int st = dictproj_layer_file_info(path, &k, &d_out, &total);
  if (st) return st;
  if (k <= 0 || k % 16 || k > 65535 || d_out <= 0 || total % 16) return fail(DICTPROJ_ERR_VALUE, "layer_load: bad shape in file");
  const size_t nseg = (size_t)(k + 255) / 256;
  std::vector<uint32_t> col_ptr((size_t)d_out + 1);
  std::vector<uint8_t> codes(total / 2), scales(total / 16), idx(total);
  std::vector<uint16_t> ss((size_t)d_out * nseg);
  float s = 0.0f;
  if ((st = dictproj_layer_file_read(path, col_ptr.data(), codes.data(), scales.data(), idx.data(), ss.data(), &s, k,
                                     d_out, total)))
    return st;
  return dictproj_layer_upload(col_ptr.data(), codes.data(), scales.data(), idx.data(), ss.data(), s, k, d_out, out);
}

}  // extern "C"
