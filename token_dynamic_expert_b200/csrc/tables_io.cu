// tables_io.cu -- the offline tables ([ACE] "Methodology 1" and
// "Methodology 2": A^GSP, A^RCR, their maximum, and the singular values of
// the bound) kept in a file, so that a table build done once can be reloaded
// instead of recomputed.  The tables are checkpoint-preserving and depend only on
// the frozen weights ([ACE] "Practical Implications").  Host code only.
//
// File layout, little-endian:
//   offset  0  8 bytes  magic "ACETBL\0\x01"
//   offset  8  u32      format version (1)
//   offset 12  u32      n_layers
//   offset 16  u32      E (experts per layer)
//   offset 20  u32      flags: bit 0 set when sigma is present
//   offset 24  u64      FNV-1a 64-bit hash of the payload bytes
//   offset 32  payload: fp32 a_gsp [L][E], a_rcr [L][E], amax [L][E],
//              then sigma [L][E][3] when present
// A file is written under a temporary name and renamed into place, so a
// crash mid-write leaves the previous file (or none), never a torn one.
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <string>
#include <vector>

#include "ace_internal.h"

namespace {

const unsigned char kMagic[8] = {'A', 'C', 'E', 'T', 'B', 'L', 0, 1};
constexpr uint32_t kVersion = 1;
constexpr size_t kHeader = 32;
constexpr int kMaxLayers = 1 << 16;

uint64_t fnv1a(const unsigned char* p, size_t n, uint64_t h) {
  for (size_t i = 0; i < n; ++i) {
    h ^= p[i];
    h *= 1099511628211ull;
  }
  return h;
}

void put32(unsigned char* p, uint32_t v) {
  for (int i = 0; i < 4; ++i) p[i] = (unsigned char)(v >> (8 * i));
}
void put64(unsigned char* p, uint64_t v) {
  for (int i = 0; i < 8; ++i) p[i] = (unsigned char)(v >> (8 * i));
}
uint32_t get32(const unsigned char* p) {
  uint32_t v = 0;
  for (int i = 0; i < 4; ++i) v |= (uint32_t)p[i] << (8 * i);
  return v;
}
uint64_t get64(const unsigned char* p) {
  uint64_t v = 0;
  for (int i = 0; i < 8; ++i) v |= (uint64_t)p[i] << (8 * i);
  return v;
}

// fp32 arrays as little-endian bytes (the host is little-endian on every
// platform CUDA supports; the byte copy keeps the file format explicit)
void append_f32(std::vector<unsigned char>& out, const float* a, size_t n) {
  const size_t at = out.size();
  out.resize(at + n * 4);
  memcpy(out.data() + at, a, n * 4);
}

struct Header {
  uint32_t version, n_layers, E, flags;
  uint64_t hash;
};

// Reads and checks the header and the payload size; the payload stays in `buf`.
ace_status read_file(const char* path, Header* h, std::vector<unsigned char>* buf) {
  if (!path) return ACE_ERR_INVALID_ARG;
  FILE* f = fopen(path, "rb");
  if (!f) return ACE_ERR_IO;
  unsigned char hd[kHeader];
  if (fread(hd, 1, kHeader, f) != kHeader || memcmp(hd, kMagic, 8) != 0) {
    fclose(f);
    return ACE_ERR_IO;
  }
  h->version = get32(hd + 8);
  h->n_layers = get32(hd + 12);
  h->E = get32(hd + 16);
  h->flags = get32(hd + 20);
  h->hash = get64(hd + 24);
  if (h->version != kVersion || h->n_layers < 1 || h->n_layers > (uint32_t)kMaxLayers ||
      h->E < 1 || h->E > (uint32_t)ace::kMaxE || (h->flags & ~1u) != 0) {
    fclose(f);
    return ACE_ERR_IO;
  }
  const size_t le = (size_t)h->n_layers * h->E;
  const size_t payload = le * 4 * (3 + ((h->flags & 1u) ? 3 : 0));
  buf->resize(payload + 1);
  const size_t got = fread(buf->data(), 1, payload + 1, f);  // one byte more: detects trailing data
  fclose(f);
  if (got != payload) return ACE_ERR_IO;
  buf->resize(payload);
  if (fnv1a(buf->data(), payload, 14695981039346656037ull) != h->hash) return ACE_ERR_IO;
  return ACE_OK;
}

}  // namespace

extern "C" {

ace_status ace_tables_save(const char* path, int n_layers, int E, const float* a_gsp,
                           const float* a_rcr, const float* amax, const float* sigma) {
  if (!path || n_layers < 1 || n_layers > kMaxLayers || E < 1 || E > ace::kMaxE || !a_gsp ||
      !a_rcr || !amax)
    return ACE_ERR_INVALID_ARG;
  const size_t le = (size_t)n_layers * E;
  std::vector<unsigned char> buf(kHeader);
  append_f32(buf, a_gsp, le);
  append_f32(buf, a_rcr, le);
  append_f32(buf, amax, le);
  if (sigma) append_f32(buf, sigma, le * 3);
  memcpy(buf.data(), kMagic, 8);
  put32(buf.data() + 8, kVersion);
  put32(buf.data() + 12, (uint32_t)n_layers);
  put32(buf.data() + 16, (uint32_t)E);
  put32(buf.data() + 20, sigma ? 1u : 0u);
  put64(buf.data() + 24, fnv1a(buf.data() + kHeader, buf.size() - kHeader, 14695981039346656037ull));
  const std::string tmp = std::string(path) + ".tmp";
  FILE* f = fopen(tmp.c_str(), "wb");
  if (!f) return ACE_ERR_IO;
  const bool ok = fwrite(buf.data(), 1, buf.size(), f) == buf.size();
  const bool closed = fclose(f) == 0;
  if (!ok || !closed || rename(tmp.c_str(), path) != 0) {
    remove(tmp.c_str());
    return ACE_ERR_IO;
  }
  return ACE_OK;
}

ace_status ace_tables_info(const char* path, int* n_layers, int* E, int* has_sigma) {
  Header h;
  std::vector<unsigned char> buf;
  const ace_status st = read_file(path, &h, &buf);
  if (st != ACE_OK) return st;
  if (n_layers) *n_layers = (int)h.n_layers;
  if (E) *E = (int)h.E;
  if (has_sigma) *has_sigma = (int)(h.flags & 1u);
  return ACE_OK;
}

ace_status ace_tables_load(const char* path, int n_layers, int E, float* a_gsp, float* a_rcr,
                           float* amax, float* sigma) {
  if (!a_gsp || !a_rcr || !amax) return ACE_ERR_INVALID_ARG;
  Header h;
  std::vector<unsigned char> buf;
  const ace_status st = read_file(path, &h, &buf);
  if (st != ACE_OK) return st;
  if ((int)h.n_layers != n_layers || (int)h.E != E) return ACE_ERR_INVALID_ARG;
  if (sigma && !(h.flags & 1u)) return ACE_ERR_INVALID_ARG;
  const size_t le = (size_t)n_layers * E;
  memcpy(a_gsp, buf.data(), le * 4);
  memcpy(a_rcr, buf.data() + le * 4, le * 4);
  memcpy(amax, buf.data() + 2 * le * 4, le * 4);
  if (sigma) memcpy(sigma, buf.data() + 3 * le * 4, le * 12);
  return ACE_OK;
}

}  // extern "C"
