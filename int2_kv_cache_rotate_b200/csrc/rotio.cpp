// Rotation files: the calibrated U_K and U_V of every layer of a model, so
// that a deployment loads precomputed rotations instead of calibrating
// (gen-hub.ru, "Together AI открывает OSCAR…", section "Открытый код — это
// серьёзно": rotations are computed offline, once, and shipped per model;
// aiforradalom.hu, section "OSCAR: figyelem-tudatos és bevetésre kész": a
// set of precomputed rotations for the supported models).  The pages give no
// file format; this one is the library's own (layout in okv.h).
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <vector>

#include "okv.h"
#include "okv_internal.h"

namespace {

constexpr char kMagic[8] = {'O', 'K', 'V', 'R', 'O', 'T', 'S', '1'};
constexpr uint32_t kFormatVersion = 1;
constexpr uint32_t kMaxTag = 4096;

// 64-bit FNV-1a over a byte range, continuing from h
uint64_t fnv1a(uint64_t h, const void* p, size_t n) {
  const unsigned char* b = static_cast<const unsigned char*>(p);
  for (size_t i = 0; i < n; ++i) {
    h ^= b[i];
    h *= 0x100000001b3ull;
  }
  return h;
}
constexpr uint64_t kFnvBasis = 0xcbf29ce484222325ull;

struct Header {
  char magic[8];
  uint32_t version, d, num_layers, num_kv_heads, tag_len, reserved;
};
static_assert(sizeof(Header) == 32, "packed header");

struct File {
  FILE* f = nullptr;
  ~File() {
    if (f != nullptr) fclose(f);
  }
};

// max |U^T U - I| over the n x n matrix u (fp32, row-major), in fp64
double orthogonality_error(const float* u, int n) {
  double worst = 0.0;
  for (int i = 0; i < n; ++i)
    for (int j = i; j < n; ++j) {
      double s = 0.0;
      for (int k = 0; k < n; ++k) s += (double)u[(size_t)k * n + i] * (double)u[(size_t)k * n + j];
      worst = std::max(worst, std::fabs(s - (i == j ? 1.0 : 0.0)));
    }
  return worst;
}

}  // namespace

using okv::fail;

okv_status okv_save_rotations(const char* path, int32_t num_layers, int32_t num_kv_heads, int32_t d,
                              const float* u_k, const float* u_v, const char* tag) {
  if (path == nullptr || u_k == nullptr || u_v == nullptr)
    return fail(OKV_ERR_INVALID_ARG, "save_rotations: NULL path or matrices");
  if (num_layers < 1 || num_kv_heads < 1) return fail(OKV_ERR_INVALID_ARG, "save_rotations: empty shape");
  if (d != OKV_HEAD_DIM) return fail(OKV_ERR_UNSUPPORTED, "save_rotations: d must be %d", OKV_HEAD_DIM);
  const size_t tag_len = tag == nullptr ? 0 : strlen(tag);
  if (tag_len > kMaxTag) return fail(OKV_ERR_INVALID_ARG, "save_rotations: tag longer than %u bytes", kMaxTag);
  Header h;
  memcpy(h.magic, kMagic, 8);
  h.version = kFormatVersion;
  h.d = (uint32_t)d;
  h.num_layers = (uint32_t)num_layers;
  h.num_kv_heads = (uint32_t)num_kv_heads;
  h.tag_len = (uint32_t)tag_len;
  h.reserved = 0;
  const size_t per = (size_t)num_layers * num_kv_heads * d * d;
  uint64_t sum = fnv1a(kFnvBasis, &h, sizeof(h));
  sum = fnv1a(sum, tag, tag_len);
  sum = fnv1a(sum, u_k, per * sizeof(float));
  sum = fnv1a(sum, u_v, per * sizeof(float));
  File file;
  file.f = fopen(path, "wb");
  if (file.f == nullptr) return fail(OKV_ERR_IO, "save_rotations: cannot open %s for writing", path);
  bool ok = fwrite(&h, sizeof(h), 1, file.f) == 1;
  ok = ok && (tag_len == 0 || fwrite(tag, 1, tag_len, file.f) == tag_len);
  ok = ok && fwrite(u_k, sizeof(float), per, file.f) == per;
  ok = ok && fwrite(u_v, sizeof(float), per, file.f) == per;
  ok = ok && fwrite(&sum, sizeof(sum), 1, file.f) == 1;
  ok = (fclose(file.f) == 0) && ok;
  file.f = nullptr;
  if (!ok) return fail(OKV_ERR_IO, "save_rotations: write to %s failed", path);
  return OKV_OK;
}

okv_status okv_rotations_file_shape(const char* path, int32_t* num_layers, int32_t* num_kv_heads, int32_t* d,
                                    int32_t* tag_len) {
  if (path == nullptr) return fail(OKV_ERR_INVALID_ARG, "rotations_file_shape: NULL path");
  File file;
  file.f = fopen(path, "rb");
  if (file.f == nullptr) return fail(OKV_ERR_IO, "rotations file %s: cannot open", path);
  Header h;
  if (fread(&h, sizeof(h), 1, file.f) != 1) return fail(OKV_ERR_IO, "rotations file %s: truncated header", path);
  if (memcmp(h.magic, kMagic, 8) != 0) return fail(OKV_ERR_IO, "rotations file %s: not a rotations file", path);
  if (h.version != kFormatVersion)
    return fail(OKV_ERR_UNSUPPORTED, "rotations file %s: format version %u", path, h.version);
  if (num_layers != nullptr) *num_layers = (int32_t)h.num_layers;
  if (num_kv_heads != nullptr) *num_kv_heads = (int32_t)h.num_kv_heads;
  if (d != nullptr) *d = (int32_t)h.d;
  if (tag_len != nullptr) *tag_len = (int32_t)h.tag_len;
  return OKV_OK;
}

okv_status okv_load_rotations(const char* path, int32_t num_layers, int32_t num_kv_heads, int32_t d, float* u_k,
                              float* u_v, char* tag, size_t tag_capacity, int32_t verify) {
  if (path == nullptr || u_k == nullptr || u_v == nullptr)
    return fail(OKV_ERR_INVALID_ARG, "load_rotations: NULL path or output");
  File file;
  file.f = fopen(path, "rb");
  if (file.f == nullptr) return fail(OKV_ERR_IO, "rotations file %s: cannot open", path);
  Header h;
  if (fread(&h, sizeof(h), 1, file.f) != 1) return fail(OKV_ERR_IO, "rotations file %s: truncated header", path);
  if (memcmp(h.magic, kMagic, 8) != 0) return fail(OKV_ERR_IO, "rotations file %s: not a rotations file", path);
  if (h.version != kFormatVersion)
    return fail(OKV_ERR_UNSUPPORTED, "rotations file %s: format version %u", path, h.version);
  if ((int32_t)h.num_layers != num_layers || (int32_t)h.num_kv_heads != num_kv_heads || (int32_t)h.d != d)
    return fail(OKV_ERR_INVALID_ARG, "rotations file %s holds %u layers x %u KV heads x d=%u, not %d x %d x %d",
                path, h.num_layers, h.num_kv_heads, h.d, num_layers, num_kv_heads, d);
  if (h.tag_len > kMaxTag) return fail(OKV_ERR_IO, "rotations file %s: corrupt tag length", path);
  std::vector<char> tagbuf(h.tag_len);
  if (h.tag_len > 0 && fread(tagbuf.data(), 1, h.tag_len, file.f) != h.tag_len)
    return fail(OKV_ERR_IO, "rotations file %s: truncated", path);
  const size_t per = (size_t)num_layers * num_kv_heads * d * d;
  uint64_t stored = 0;
  if (fread(u_k, sizeof(float), per, file.f) != per || fread(u_v, sizeof(float), per, file.f) != per ||
      fread(&stored, sizeof(stored), 1, file.f) != 1)
    return fail(OKV_ERR_IO, "rotations file %s: truncated", path);
  char extra;
  if (fread(&extra, 1, 1, file.f) != 0) return fail(OKV_ERR_IO, "rotations file %s: trailing bytes", path);
  uint64_t sum = fnv1a(kFnvBasis, &h, sizeof(h));
  sum = fnv1a(sum, tagbuf.data(), tagbuf.size());
  sum = fnv1a(sum, u_k, per * sizeof(float));
  sum = fnv1a(sum, u_v, per * sizeof(float));
  if (sum != stored) return fail(OKV_ERR_IO, "rotations file %s: checksum mismatch", path);
  if (tag != nullptr && tag_capacity > 0) {
    const size_t n = std::min(tag_capacity - 1, tagbuf.size());
    memcpy(tag, tagbuf.data(), n);
    tag[n] = '\0';
  }
  if (verify) {
    for (int kind = 0; kind < 2; ++kind)
      for (size_t m = 0; m < (size_t)num_layers * num_kv_heads; ++m)
        if (orthogonality_error((kind ? u_v : u_k) + m * d * d, d) > 1e-4)
          return fail(OKV_ERR_NUMERIC, "rotations file %s: %s %zu (layer %zu, KV head %zu) is not orthogonal", path,
                      kind ? "U_V" : "U_K", m, m / num_kv_heads, m % num_kv_heads);
  }
  return OKV_OK;
}
