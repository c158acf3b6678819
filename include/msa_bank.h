/* Bank persistence and append: a pooled memory bank written to and read from one raw
 * binary file, and the re-layout that lets new documents be appended to a resident bank
 * without re-encoding the old ones.
 *
 * Defined by: "【MSA】突破100M Token 上下文：记忆稀疏注意力架构深度解析", section 8.3 (documents
 * are encoded once into K̄/V̄/K̄ᵣ, saved to a memory file and loaded by the engine for later
 * inference); "把一亿 token 装进模型的“记忆”里…", section 5.2 (the bank is encoded offline per
 * version; since the lower layers treat documents independently, new documents can be
 * encoded on their own and appended).  The pages do not give a file format: this one is
 * this library's own.
 *
 * File format (little-endian; version 1):
 *   bytes [0, 256)  header:
 *     char     magic[8] = "MSABANK1"
 *     uint32   version = 1, header_bytes = 256
 *     int32    n_layers, n_heads, head_dim, block_tokens
 *     int64    n_docs, n_blocks
 *     uint32   fields (MSA_BANK_* bits of the array sections present), reserved (0)
 *     5 x { uint64 file_offset, uint64 bytes, uint64 checksum }   section table, in order:
 *       0 doc_chunk_offsets  int64 [n_docs + 1]                (always present)
 *       1 MSA_BANK_KR        bf16  [n_layers][n_blocks][n_heads][head_dim]  unit routing keys
 *       2 MSA_BANK_KR_F8     E4M3  [n_layers][n_blocks][n_heads][head_dim]  filter copy
 *       3 MSA_BANK_KV        bf16  [n_layers][n_blocks][2][n_heads][head_dim] content K̄, V̄
 *       4 MSA_BANK_NORM      fp32  [n_layers][n_blocks][n_heads]  routing-key norms
 *     (absent sections have offset, bytes and checksum 0), zero padding to 256.
 *   Each section starts at a multiple of 4096 bytes, zero padding between sections.
 *   checksum of a section: its bytes zero-padded to a multiple of 32 and read as uint64
 *   words w[0..n); four lanes h_j = 0xcbf29ce484222325 ^ j (j = 0..3) take the words
 *   w[4i + j] in order as h_j = (h_j ^ w) * 0x100000001b3 (mod 2^64); the checksum is
 *   h_0 ^ rotl(h_1, 16) ^ rotl(h_2, 32) ^ rotl(h_3, 48).
 *
 * Arrays may be device or host pointers (told apart by cudaPointerGetAttributes; with no
 * CUDA device every pointer is host).  Device arrays move through the caller's staging
 * buffer (page-locked host memory of at least 2 MB, used as two halves so copies overlap
 * the file I/O); host arrays are read and written directly.  Save and load block the
 * calling thread until the file and the destination arrays are complete; `stream` orders
 * their device copies after earlier work on it.  Errors: MSA_ERR_INVALID_ARG (null or
 * inconsistent arguments), MSA_ERR_IO (the file cannot be opened, read or written, a bad
 * magic or version, a size that disagrees with the header, a checksum mismatch),
 * MSA_ERR_CUDA (a copy failed).
 */
#ifndef MSA_BANK_H
#define MSA_BANK_H

#include "msa_common.h"

#ifdef __cplusplus
extern "C" {
#endif

#define MSA_BANK_KR 1u
#define MSA_BANK_KR_F8 2u
#define MSA_BANK_KV 4u
#define MSA_BANK_NORM 8u

typedef struct msa_bank_info {
  int32_t n_layers, n_heads, head_dim, block_tokens;
  int64_t n_docs, n_blocks;
  uint32_t fields; /* MSA_BANK_* bits */
} msa_bank_info;

/* Writes a bank file.  doc_chunk_offsets: HOST int64 [n_docs + 1] (0, ..., n_blocks,
 * non-decreasing).  kr_hat, kr_f8, content_kv, kr_norm: the arrays named by info->fields
 * (others ignored, may be NULL), layouts as in the section table. */
msa_status msa_bank_save(const char* path, const msa_bank_info* info, const int64_t* doc_chunk_offsets,
                         const void* kr_hat, const void* kr_f8, const void* content_kv, const void* kr_norm,
                         void* staging, size_t staging_bytes, msa_stream_t stream);

/* Reads a bank file's header into *info (no array data). */
msa_status msa_bank_read_info(const char* path, msa_bank_info* info);

/* Reads a bank file into caller arrays sized from msa_bank_read_info.  doc_chunk_offsets:
 * HOST int64 [n_docs + 1].  For each section present in the file whose destination is
 * non-NULL the data is loaded and its checksum verified; a NULL destination skips the
 * section.  A destination given for a section the file lacks is MSA_ERR_INVALID_ARG. */
msa_status msa_bank_load(const char* path, int64_t* doc_chunk_offsets, void* kr_hat, void* kr_f8,
                         void* content_kv, void* kr_norm, void* staging, size_t staging_bytes,
                         msa_stream_t stream);

/* Append support.  Copies rows [0, rows_old) of each of n_layers layers of src
 * ([n_layers][rows_old][row_bytes]) into dst ([n_layers][rows_new][row_bytes], rows_new >=
 * rows_old), leaving rows [rows_old, rows_new) of every layer for the new documents' blocks
 * (written afterwards by msa_pool_blocks / msa_route_filter_keys).  One copy per layer on
 * `stream` when either pointer is device memory (dst must not overlap src); between two
 * host arrays plain copies done on return, top layer first, so dst may be src itself
 * grown in place. */
msa_status msa_bank_relayout(const void* src, void* dst, int32_t n_layers, int64_t rows_old, int64_t rows_new,
                             int64_t row_bytes, msa_stream_t stream);

/* Host: offsets of the bank after appending n_new documents whose own block offsets are
 * new_offsets [n_new + 1] (starting at 0) to a bank with old_offsets [n_old + 1]:
 * out [n_old + n_new + 1] = old_offsets, then old_offsets[n_old] + new_offsets[1..]. */
msa_status msa_bank_append_offsets(const int64_t* old_offsets, int64_t n_old, const int64_t* new_offsets,
                                   int64_t n_new, int64_t* out);

const char* msa_bank_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MSA_BANK_H */
