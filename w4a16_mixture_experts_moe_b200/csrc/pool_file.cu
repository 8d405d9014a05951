// The packed expert pool as a file, so the packing is done a single time
// (ExactMoE paper, Figure 1 caption: the experts are quantised and packed
// ahead of time, and the pinned host pool holds every packed expert). Host code only; no
// CUDA call is made, so a pool can be written and checked on a machine
// without a GPU.
//
// Layout (little-endian): a 64-byte header, then the records [layers][E] of
// record_bytes each, exactly as moe_quantize_pack lays them out in a bank.
//   bytes  0-7   magic "EXMOEPK1"
//   bytes  8-11  format version (1)
//   bytes 12-15  header size (64)
//   bytes 16-31  layers, E, H, I (int32 each)
//   bytes 32-39  record_bytes (int64)
//   bytes 40-47  payload bytes = layers * E * record_bytes (int64)
//   bytes 48-55  payload checksum (uint64, below)
//   bytes 56-63  zero
// Checksum: FNV-1a over the payload taken as little-endian 64-bit words
// (offset basis 0xcbf29ce484222325, prime 0x100000001b3, one xor and one
// multiply per word); payloads are multiples of 256 bytes.
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <string>

#include "common.cuh"

namespace moe {

constexpr char POOL_MAGIC[8] = {'E', 'X', 'M', 'O', 'E', 'P', 'K', '1'};
constexpr uint32_t POOL_VERSION = 1;
constexpr uint32_t POOL_HEADER = 64;

struct PoolHeader {
  char magic[8];
  uint32_t version, header_bytes;
  int32_t layers, E, H, I;
  int64_t record_bytes, payload_bytes;
  uint64_t checksum, zero;
};
static_assert(sizeof(PoolHeader) == POOL_HEADER, "pool header is 64 bytes");

struct Fnv64 {
  uint64_t h = 0xcbf29ce484222325ull;
  void words(const uint8_t *p, size_t n) {  // n a multiple of 8
    for (size_t i = 0; i < n; i += 8) {
      uint64_t w;
      memcpy(&w, p + i, 8);
      h = (h ^ w) * 0x100000001b3ull;
    }
  }
};

static int check_info(const moe_pool_info *info, const char *what) {
  if (!info) return set_error(MOE_ERR_INVALID_ARG, "%s: info is NULL", what);
  if (info->layers < 1 || info->E < 1 || info->E > MAX_E)
    return set_error(MOE_ERR_SHAPE, "%s: layers=%d E=%d", what, info->layers, info->E);
  moe_record_layout L;
  if (moe_expert_record_layout(info->H, info->I, &L) != MOE_OK) return MOE_ERR_SHAPE;
  if (info->record_bytes < L.bytes || info->record_bytes % 256)
    return set_error(MOE_ERR_SHAPE, "%s: record_bytes=%lld (need >= %lld for H=%d I=%d, multiple of 256)", what,
                     (long long)info->record_bytes, (long long)L.bytes, info->H, info->I);
  return MOE_OK;
}

static int read_header(FILE *f, const char *path, PoolHeader *h, const char *what) {
  if (fread(h, 1, sizeof(*h), f) != sizeof(*h))
    return set_error(MOE_ERR_INVALID_ARG, "%s: %s is shorter than a pool header", what, path);
  if (memcmp(h->magic, POOL_MAGIC, 8) != 0)
    return set_error(MOE_ERR_INVALID_ARG, "%s: %s is not a packed expert pool (bad magic)", what, path);
  if (h->version != POOL_VERSION || h->header_bytes != POOL_HEADER)
    return set_error(MOE_ERR_UNSUPPORTED, "%s: %s has format version %u (header %u bytes); this library reads "
                     "version %u", what, path, h->version, h->header_bytes, POOL_VERSION);
  moe_pool_info info = {h->layers, h->E, h->H, h->I, h->record_bytes};
  int st = check_info(&info, what);
  if (st != MOE_OK) return st;
  if (h->payload_bytes != int64_t(h->layers) * h->E * h->record_bytes)
    return set_error(MOE_ERR_INVALID_ARG, "%s: %s: payload size %lld does not match its shape", what, path,
                     (long long)h->payload_bytes);
  return MOE_OK;
}

}  // namespace moe

extern "C" int moe_pool_save(const char *path, const moe_pool_info *info, const void *pool) {
  moe::NvtxScope nvtx_scope("moe_pool_save");
  using namespace moe;
  if (!path || !pool) return set_error(MOE_ERR_INVALID_ARG, "moe_pool_save: NULL pointer");
  int st = check_info(info, "moe_pool_save");
  if (st != MOE_OK) return st;
  PoolHeader h;
  memset(&h, 0, sizeof(h));
  memcpy(h.magic, POOL_MAGIC, 8);
  h.version = POOL_VERSION;
  h.header_bytes = POOL_HEADER;
  h.layers = info->layers; h.E = info->E; h.H = info->H; h.I = info->I;
  h.record_bytes = info->record_bytes;
  h.payload_bytes = int64_t(info->layers) * info->E * info->record_bytes;
  const uint8_t *p = static_cast<const uint8_t *>(pool);
  Fnv64 sum;
  sum.words(p, size_t(h.payload_bytes));
  h.checksum = sum.h;
  const std::string tmp = std::string(path) + ".tmp";
  FILE *f = fopen(tmp.c_str(), "wb");
  if (!f) return set_error(MOE_ERR_INVALID_ARG, "moe_pool_save: cannot create %s", tmp.c_str());
  bool ok = fwrite(&h, 1, sizeof(h), f) == sizeof(h);
  for (int64_t off = 0; ok && off < h.payload_bytes;) {
    const size_t n = size_t(std::min<int64_t>(h.payload_bytes - off, int64_t(1) << 26));
    ok = fwrite(p + off, 1, n, f) == n;
    off += int64_t(n);
  }
  ok = (fclose(f) == 0) && ok;
  if (!ok || rename(tmp.c_str(), path) != 0) {
    remove(tmp.c_str());
    return set_error(MOE_ERR_INVALID_ARG, "moe_pool_save: writing %s failed", path);
  }
  return MOE_OK;
}

extern "C" int moe_pool_file_info(const char *path, moe_pool_info *info) {
  using namespace moe;
  if (!path || !info) return set_error(MOE_ERR_INVALID_ARG, "moe_pool_file_info: NULL pointer");
  FILE *f = fopen(path, "rb");
  if (!f) return set_error(MOE_ERR_INVALID_ARG, "moe_pool_file_info: cannot open %s", path);
  PoolHeader h;
  const int st = read_header(f, path, &h, "moe_pool_file_info");
  fclose(f);
  if (st != MOE_OK) return st;
  *info = moe_pool_info{h.layers, h.E, h.H, h.I, h.record_bytes};
  return MOE_OK;
}

extern "C" int moe_pool_load(const char *path, void *pool, size_t capacity, moe_pool_info *info) {
  moe::NvtxScope nvtx_scope("moe_pool_load");
  using namespace moe;
  if (!path || !pool) return set_error(MOE_ERR_INVALID_ARG, "moe_pool_load: NULL pointer");
  FILE *f = fopen(path, "rb");
  if (!f) return set_error(MOE_ERR_INVALID_ARG, "moe_pool_load: cannot open %s", path);
  PoolHeader h;
  int st = read_header(f, path, &h, "moe_pool_load");
  if (st != MOE_OK) { fclose(f); return st; }
  if (size_t(h.payload_bytes) > capacity) {
    fclose(f);
    return set_error(MOE_ERR_INVALID_ARG, "moe_pool_load: %s holds %lld bytes of records, the buffer %zu", path,
                     (long long)h.payload_bytes, capacity);
  }
  uint8_t *p = static_cast<uint8_t *>(pool);
  Fnv64 sum;
  bool ok = true;
  for (int64_t off = 0; ok && off < h.payload_bytes;) {
    const size_t n = size_t(std::min<int64_t>(h.payload_bytes - off, int64_t(1) << 26));
    ok = fread(p + off, 1, n, f) == n;
    if (ok) sum.words(p + off, n);
    off += int64_t(n);
  }
  const bool trailing = ok && fgetc(f) != EOF;
  fclose(f);
  if (!ok) return set_error(MOE_ERR_INVALID_ARG, "moe_pool_load: %s is truncated", path);
  if (trailing) return set_error(MOE_ERR_INVALID_ARG, "moe_pool_load: %s has bytes past its records", path);
  if (sum.h != h.checksum)
    return set_error(MOE_ERR_INVALID_ARG, "moe_pool_load: %s: checksum mismatch (the file is corrupt)", path);
  if (info) *info = moe_pool_info{h.layers, h.E, h.H, h.I, h.record_bytes};
  return MOE_OK;
}
