// Bank persistence (one raw binary file per pooled bank) and the append re-layout.
//
// Follows "【MSA】突破100M Token 上下文：记忆稀疏注意力架构深度解析", section 8.3 (encode the
// documents once, save the memory, load it for inference) and "把一亿 token 装进模型的“记忆”
// 里…", section 5.2 (documents are independent below the routing, so new ones can be
// encoded alone and appended).  The format and its checksum are defined in msa_bank.h.
// Host code only: device arrays cross through the caller's page-locked staging buffer in
// two halves, so each half's copy overlaps the file I/O of the other.
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdio.h>
#include <string.h>

#include <vector>

#include "common.cuh"
#include "msa_bank.h"

MSA_DEFINE_LAST_ERROR(msa_bank_last_error)

namespace {

constexpr char kMagic[8] = {'M', 'S', 'A', 'B', 'A', 'N', 'K', '1'};
constexpr uint32_t kVersion = 1;
constexpr uint32_t kHeaderBytes = 256;
constexpr uint64_t kAlign = 4096;
constexpr int kSections = 5;
constexpr size_t kMinStaging = 2u << 20;

struct Section {
  uint64_t offset, bytes, checksum;
};

struct Header {
  char magic[8];
  uint32_t version, header_bytes;
  int32_t n_layers, n_heads, head_dim, block_tokens;
  int64_t n_docs, n_blocks;
  uint32_t fields, reserved;
  Section sec[kSections];
};
static_assert(sizeof(Header) <= kHeaderBytes, "header fits its 256 bytes");
static_assert(offsetof(Header, n_docs) == 32 && offsetof(Header, sec) == 56, "packed as documented");

// The four-lane word checksum of msa_bank.h, fed incrementally (chunk sizes multiples of 32
// bytes except the last).
struct Checksum {
  uint64_t h[4];
  uint64_t words = 0;  // words consumed (the lane of the next word is words % 4)
  Checksum() {
    for (int j = 0; j < 4; ++j) h[j] = 0xcbf29ce484222325ull ^ (uint64_t)j;
  }
  void feed(const void* p, size_t n) {
    const unsigned char* c = static_cast<const unsigned char*>(p);
    const size_t full = n / 8;
    for (size_t i = 0; i < full; ++i) {
      uint64_t w;
      memcpy(&w, c + 8 * i, 8);
      uint64_t& x = h[(words + i) & 3];
      x = (x ^ w) * 0x100000001b3ull;
    }
    words += full;
    const size_t tail = n - 8 * full;
    if (tail) {  // the last chunk of a section: zero-pad to whole words, then to 4 words
      uint64_t w = 0;
      memcpy(&w, c + 8 * full, tail);
      uint64_t& x = h[words & 3];
      x = (x ^ w) * 0x100000001b3ull;
      ++words;
    }
  }
  uint64_t finish() {
    while (words & 3) {  // zero words up to a multiple of 32 bytes
      uint64_t& x = h[words & 3];
      x = (x ^ 0ull) * 0x100000001b3ull;
      ++words;
    }
    auto rotl = [](uint64_t v, int r) { return (v << r) | (v >> (64 - r)); };
    return h[0] ^ rotl(h[1], 16) ^ rotl(h[2], 32) ^ rotl(h[3], 48);
  }
};

uint64_t align_up(uint64_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// true when p is device memory (needs staging); false for host memory or with no device
bool is_device(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();  // (no device, or a pointer the runtime does not know: clear the error)
    return false;
  }
  return a.type == cudaMemoryTypeDevice;
}

bool section_bytes(const msa_bank_info& in, int s, uint64_t* out) {
  const uint64_t rows = (uint64_t)in.n_layers * (uint64_t)in.n_blocks;
  const uint64_t hd = (uint64_t)in.n_heads * (uint64_t)in.head_dim;
  switch (s) {
    case 0: *out = ((uint64_t)in.n_docs + 1) * 8; return true;
    case 1: *out = (in.fields & MSA_BANK_KR) ? rows * hd * 2 : 0; return true;
    case 2: *out = (in.fields & MSA_BANK_KR_F8) ? rows * hd : 0; return true;
    case 3: *out = (in.fields & MSA_BANK_KV) ? rows * hd * 4 : 0; return true;
    case 4: *out = (in.fields & MSA_BANK_NORM) ? rows * (uint64_t)in.n_heads * 4 : 0; return true;
  }
  return false;
}

bool info_ok(const msa_bank_info& in) {
  return in.n_layers >= 1 && in.n_heads >= 1 && in.head_dim >= 1 && in.block_tokens >= 1 && in.n_docs >= 0 &&
         in.n_blocks >= 0 && (in.fields & ~(MSA_BANK_KR | MSA_BANK_KR_F8 | MSA_BANK_KV | MSA_BANK_NORM)) == 0;
}

struct File {
  FILE* f = nullptr;
  ~File() {
    if (f) fclose(f);
  }
};

// Writes n bytes of src (device or host) to f, returning the checksum via ck.
msa_status write_array(FILE* f, const void* src, uint64_t n, unsigned char* stage, size_t stage_bytes,
                       cudaStream_t s, Checksum* ck) {
  if (!is_device(src)) {
    const unsigned char* p = static_cast<const unsigned char*>(src);
    const size_t step = 64u << 20;
    for (uint64_t o = 0; o < n; o += step) {
      const size_t len = (size_t)(n - o < step ? n - o : step);
      ck->feed(p + o, len);
      if (fwrite(p + o, 1, len, f) != len) return msa_fail(MSA_ERR_IO, "write failed");
    }
    return MSA_OK;
  }
  const size_t half = stage_bytes / 2 / 32 * 32;
  unsigned char* buf[2] = {stage, stage + half};
  cudaEvent_t ev[2];
  MSA_CUDA_TRY(cudaEventCreateWithFlags(&ev[0], cudaEventDisableTiming));
  if (cudaEventCreateWithFlags(&ev[1], cudaEventDisableTiming) != cudaSuccess) {
    cudaEventDestroy(ev[0]);
    return msa_fail(MSA_ERR_CUDA, "event create failed");
  }
  const uint64_t chunks = (n + half - 1) / half;
  msa_status st = MSA_OK;
  auto issue = [&](uint64_t c) -> bool {
    const uint64_t o = c * half;
    const size_t len = (size_t)(n - o < half ? n - o : half);
    return cudaMemcpyAsync(buf[c & 1], static_cast<const unsigned char*>(src) + o, len, cudaMemcpyDeviceToHost,
                           s) == cudaSuccess &&
           cudaEventRecord(ev[c & 1], s) == cudaSuccess;
  };
  if (chunks > 0 && !issue(0)) st = msa_fail(MSA_ERR_CUDA, "device-to-host copy failed");
  for (uint64_t c = 0; c < chunks && st == MSA_OK; ++c) {
    if (c + 1 < chunks && !issue(c + 1)) {  // the other half was written out last iteration
      st = msa_fail(MSA_ERR_CUDA, "device-to-host copy failed");
      break;
    }
    if (cudaEventSynchronize(ev[c & 1]) != cudaSuccess) {
      st = msa_fail(MSA_ERR_CUDA, "device-to-host copy failed");
      break;
    }
    const uint64_t o = c * half;
    const size_t len = (size_t)(n - o < half ? n - o : half);
    ck->feed(buf[c & 1], len);
    if (fwrite(buf[c & 1], 1, len, f) != len) st = msa_fail(MSA_ERR_IO, "write failed");
  }
  cudaEventSynchronize(ev[0]);
  cudaEventSynchronize(ev[1]);
  cudaEventDestroy(ev[0]);
  cudaEventDestroy(ev[1]);
  return st;
}

// Reads n bytes from f into dst (device or host), returning the checksum via ck.
msa_status read_array(FILE* f, void* dst, uint64_t n, unsigned char* stage, size_t stage_bytes, cudaStream_t s,
                      Checksum* ck) {
  if (!is_device(dst)) {
    unsigned char* p = static_cast<unsigned char*>(dst);
    const size_t step = 64u << 20;
    for (uint64_t o = 0; o < n; o += step) {
      const size_t len = (size_t)(n - o < step ? n - o : step);
      if (fread(p + o, 1, len, f) != len) return msa_fail(MSA_ERR_IO, "file shorter than its header states");
      ck->feed(p + o, len);
    }
    return MSA_OK;
  }
  const size_t half = stage_bytes / 2 / 32 * 32;
  unsigned char* buf[2] = {stage, stage + half};
  cudaEvent_t ev[2];
  MSA_CUDA_TRY(cudaEventCreateWithFlags(&ev[0], cudaEventDisableTiming));
  if (cudaEventCreateWithFlags(&ev[1], cudaEventDisableTiming) != cudaSuccess) {
    cudaEventDestroy(ev[0]);
    return msa_fail(MSA_ERR_CUDA, "event create failed");
  }
  bool used[2] = {false, false};
  msa_status st = MSA_OK;
  for (uint64_t o = 0, c = 0; o < n && st == MSA_OK; o += half, ++c) {
    const int b = (int)(c & 1);
    if (used[b] && cudaEventSynchronize(ev[b]) != cudaSuccess) {  // its previous copy has left
      st = msa_fail(MSA_ERR_CUDA, "host-to-device copy failed");
      break;
    }
    const size_t len = (size_t)(n - o < half ? n - o : half);
    if (fread(buf[b], 1, len, f) != len) {
      st = msa_fail(MSA_ERR_IO, "file shorter than its header states");
      break;
    }
    ck->feed(buf[b], len);
    if (cudaMemcpyAsync(static_cast<unsigned char*>(dst) + o, buf[b], len, cudaMemcpyHostToDevice, s) !=
            cudaSuccess ||
        cudaEventRecord(ev[b], s) != cudaSuccess) {
      st = msa_fail(MSA_ERR_CUDA, "host-to-device copy failed");
      break;
    }
    used[b] = true;
  }
  for (int b = 0; b < 2; ++b)
    if (used[b] && cudaEventSynchronize(ev[b]) != cudaSuccess && st == MSA_OK)
      st = msa_fail(MSA_ERR_CUDA, "host-to-device copy failed");
  cudaEventDestroy(ev[0]);
  cudaEventDestroy(ev[1]);
  return st;
}

bool pad_to(FILE* f, uint64_t target) {
  long cur = ftell(f);
  if (cur < 0 || (uint64_t)cur > target) return false;
  static const unsigned char zeros[4096] = {0};
  uint64_t left = target - (uint64_t)cur;
  while (left) {
    const size_t n = (size_t)(left < sizeof(zeros) ? left : sizeof(zeros));
    if (fwrite(zeros, 1, n, f) != n) return false;
    left -= n;
  }
  return true;
}

msa_status read_header(FILE* f, Header* h) {
  unsigned char raw[kHeaderBytes];
  if (fread(raw, 1, kHeaderBytes, f) != kHeaderBytes) return msa_fail(MSA_ERR_IO, "file shorter than a header");
  memcpy(h, raw, sizeof(Header));
  if (memcmp(h->magic, kMagic, 8) != 0) return msa_fail(MSA_ERR_IO, "not a bank file (magic)");
  if (h->version != kVersion || h->header_bytes != kHeaderBytes)
    return msa_fail(MSA_ERR_IO, "unsupported bank file version %u", h->version);
  msa_bank_info in{h->n_layers, h->n_heads, h->head_dim, h->block_tokens, h->n_docs, h->n_blocks, h->fields};
  if (!info_ok(in)) return msa_fail(MSA_ERR_IO, "bank file header out of range");
  for (int s = 0; s < kSections; ++s) {
    uint64_t want = 0;
    section_bytes(in, s, &want);
    if (h->sec[s].bytes != want) return msa_fail(MSA_ERR_IO, "section %d size disagrees with the header", s);
    if (want && (h->sec[s].offset % kAlign) != 0) return msa_fail(MSA_ERR_IO, "section %d misaligned", s);
  }
  return MSA_OK;
}

}  // namespace

extern "C" msa_status msa_bank_save(const char* path, const msa_bank_info* info, const int64_t* doc_chunk_offsets,
                                    const void* kr_hat, const void* kr_f8, const void* content_kv,
                                    const void* kr_norm, void* staging, size_t staging_bytes, msa_stream_t stream) {
  if (!path || !info || !doc_chunk_offsets) return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  if (!info_ok(*info)) return msa_fail(MSA_ERR_INVALID_ARG, "bank sizes or fields out of range");
  const void* arr[kSections] = {doc_chunk_offsets, kr_hat, kr_f8, content_kv, kr_norm};
  const uint32_t bit[kSections] = {0, MSA_BANK_KR, MSA_BANK_KR_F8, MSA_BANK_KV, MSA_BANK_NORM};
  bool any_device = false;
  for (int s = 1; s < kSections; ++s) {
    if ((info->fields & bit[s]) && !arr[s]) return msa_fail(MSA_ERR_INVALID_ARG, "array of field %u is null", bit[s]);
    if ((info->fields & bit[s]) && is_device(arr[s])) any_device = true;
  }
  if (any_device && (!staging || staging_bytes < kMinStaging))
    return msa_fail(MSA_ERR_INVALID_ARG, "device arrays need a staging buffer of at least 2 MB");
  if (doc_chunk_offsets[0] != 0 || doc_chunk_offsets[info->n_docs] != info->n_blocks)
    return msa_fail(MSA_ERR_INVALID_ARG, "doc_chunk_offsets must run from 0 to n_blocks");
  for (int64_t d = 0; d < info->n_docs; ++d)
    if (doc_chunk_offsets[d + 1] < doc_chunk_offsets[d])
      return msa_fail(MSA_ERR_INVALID_ARG, "doc_chunk_offsets decrease at %lld", (long long)d);

  Header h;
  memset(&h, 0, sizeof(h));
  memcpy(h.magic, kMagic, 8);
  h.version = kVersion;
  h.header_bytes = kHeaderBytes;
  h.n_layers = info->n_layers;
  h.n_heads = info->n_heads;
  h.head_dim = info->head_dim;
  h.block_tokens = info->block_tokens;
  h.n_docs = info->n_docs;
  h.n_blocks = info->n_blocks;
  h.fields = info->fields;
  uint64_t pos = kAlign;
  for (int s = 0; s < kSections; ++s) {
    section_bytes(*info, s, &h.sec[s].bytes);
    if (h.sec[s].bytes) {
      h.sec[s].offset = pos;
      pos = align_up(pos + h.sec[s].bytes);
    }
  }
  File f;
  f.f = fopen(path, "wb");
  if (!f.f) return msa_fail(MSA_ERR_IO, "cannot open %s for writing", path);
  unsigned char raw[kHeaderBytes];
  memset(raw, 0, sizeof(raw));
  if (fwrite(raw, 1, kHeaderBytes, f.f) != kHeaderBytes) return msa_fail(MSA_ERR_IO, "write failed");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (int i = 0; i < kSections; ++i) {
    if (!h.sec[i].bytes) continue;
    if (!pad_to(f.f, h.sec[i].offset)) return msa_fail(MSA_ERR_IO, "write failed");
    Checksum ck;
    const msa_status st = write_array(f.f, arr[i], h.sec[i].bytes, static_cast<unsigned char*>(staging),
                                      staging_bytes, s, &ck);
    if (st != MSA_OK) return st;
    h.sec[i].checksum = ck.finish();
  }
  memcpy(raw, &h, sizeof(h));
  if (fseek(f.f, 0, SEEK_SET) != 0 || fwrite(raw, 1, kHeaderBytes, f.f) != kHeaderBytes)
    return msa_fail(MSA_ERR_IO, "write failed");
  if (fflush(f.f) != 0) return msa_fail(MSA_ERR_IO, "write failed");
  if (fclose(f.f) != 0) {
    f.f = nullptr;
    return msa_fail(MSA_ERR_IO, "close failed");
  }
  f.f = nullptr;
  return msa_ok();
}

extern "C" msa_status msa_bank_read_info(const char* path, msa_bank_info* info) {
  if (!path || !info) return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  File f;
  f.f = fopen(path, "rb");
  if (!f.f) return msa_fail(MSA_ERR_IO, "cannot open %s", path);
  Header h;
  const msa_status st = read_header(f.f, &h);
  if (st != MSA_OK) return st;
  *info = msa_bank_info{h.n_layers, h.n_heads, h.head_dim, h.block_tokens, h.n_docs, h.n_blocks, h.fields};
  return msa_ok();
}

extern "C" msa_status msa_bank_load(const char* path, int64_t* doc_chunk_offsets, void* kr_hat, void* kr_f8,
                                    void* content_kv, void* kr_norm, void* staging, size_t staging_bytes,
                                    msa_stream_t stream) {
  if (!path || !doc_chunk_offsets) return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  File f;
  f.f = fopen(path, "rb");
  if (!f.f) return msa_fail(MSA_ERR_IO, "cannot open %s", path);
  Header h;
  msa_status st = read_header(f.f, &h);
  if (st != MSA_OK) return st;
  void* arr[kSections] = {doc_chunk_offsets, kr_hat, kr_f8, content_kv, kr_norm};
  const uint32_t bit[kSections] = {0, MSA_BANK_KR, MSA_BANK_KR_F8, MSA_BANK_KV, MSA_BANK_NORM};
  bool any_device = false;
  for (int i = 1; i < kSections; ++i) {
    if (arr[i] && !(h.fields & bit[i])) return msa_fail(MSA_ERR_INVALID_ARG, "the file has no section %d", i);
    if (arr[i] && is_device(arr[i])) any_device = true;
  }
  if (any_device && (!staging || staging_bytes < kMinStaging))
    return msa_fail(MSA_ERR_INVALID_ARG, "device arrays need a staging buffer of at least 2 MB");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (int i = 0; i < kSections; ++i) {
    if (!arr[i] || !h.sec[i].bytes) continue;
    if (fseek(f.f, (long)h.sec[i].offset, SEEK_SET) != 0) return msa_fail(MSA_ERR_IO, "seek failed");
    Checksum ck;
    st = read_array(f.f, arr[i], h.sec[i].bytes, static_cast<unsigned char*>(staging), staging_bytes, s, &ck);
    if (st != MSA_OK) return st;
    if (ck.finish() != h.sec[i].checksum) return msa_fail(MSA_ERR_IO, "section %d checksum mismatch", i);
  }
  const int64_t* off = doc_chunk_offsets;
  if (off[0] != 0 || off[h.n_docs] != h.n_blocks) return msa_fail(MSA_ERR_IO, "stored offsets disagree with header");
  for (int64_t d = 0; d < h.n_docs; ++d)
    if (off[d + 1] < off[d]) return msa_fail(MSA_ERR_IO, "stored offsets decrease");
  return msa_ok();
}

extern "C" msa_status msa_bank_relayout(const void* src, void* dst, int32_t n_layers, int64_t rows_old,
                                        int64_t rows_new, int64_t row_bytes, msa_stream_t stream) {
  if (n_layers < 1 || rows_old < 0 || rows_new < rows_old || row_bytes < 1)
    return msa_fail(MSA_ERR_INVALID_ARG, "need n_layers >= 1, 0 <= rows_old <= rows_new, row_bytes >= 1");
  if (rows_old == 0) return msa_ok();  // nothing to copy (an empty bank may have no storage)
  if (!src || !dst) return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  const size_t width = (size_t)(rows_old * row_bytes);
  const unsigned char* a = static_cast<const unsigned char*>(src);
  unsigned char* b = static_cast<unsigned char*>(dst);
  if (!is_device(src) && !is_device(dst)) {  // host to host: plain copies, done on return
    for (int32_t l = n_layers - 1; l >= 0; --l)  // from the top down, so dst may alias src
      memmove(b + (size_t)l * (size_t)(rows_new * row_bytes), a + (size_t)l * width, width);
    return msa_ok();
  }
  // one copy per layer (a layer of a large bank exceeds the 2-D copy's pitch limit)
  for (int32_t l = 0; l < n_layers; ++l)
    MSA_CUDA_TRY(cudaMemcpyAsync(b + (size_t)l * (size_t)(rows_new * row_bytes), a + (size_t)l * width, width,
                                 cudaMemcpyDefault, reinterpret_cast<cudaStream_t>(stream)));
  return msa_ok();
}

extern "C" msa_status msa_bank_append_offsets(const int64_t* old_offsets, int64_t n_old, const int64_t* new_offsets,
                                              int64_t n_new, int64_t* out) {
  if (!old_offsets || !new_offsets || !out) return msa_fail(MSA_ERR_INVALID_ARG, "null pointer");
  if (n_old < 0 || n_new < 0 || old_offsets[0] != 0 || new_offsets[0] != 0)
    return msa_fail(MSA_ERR_INVALID_ARG, "offsets must start at 0");
  for (int64_t d = 0; d < n_old; ++d)
    if (old_offsets[d + 1] < old_offsets[d]) return msa_fail(MSA_ERR_INVALID_ARG, "old offsets decrease");
  for (int64_t d = 0; d < n_new; ++d)
    if (new_offsets[d + 1] < new_offsets[d]) return msa_fail(MSA_ERR_INVALID_ARG, "new offsets decrease");
  const int64_t base = old_offsets[n_old];
  std::vector<int64_t> tmp((size_t)(n_old + n_new + 1));  // out may alias an input
  for (int64_t d = 0; d <= n_old; ++d) tmp[(size_t)d] = old_offsets[d];
  for (int64_t d = 1; d <= n_new; ++d) tmp[(size_t)(n_old + d)] = base + new_offsets[d];
  memcpy(out, tmp.data(), tmp.size() * sizeof(int64_t));
  return msa_ok();
}
