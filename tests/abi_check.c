/* Calls every entry point of the six libraries through the prototypes of the headers in include/
 * (dlsym + __typeof__ of the declaration), with arguments the documented host-side checks
 * must reject, on a machine with or without a GPU.  Prints one line per failure and exits
 * non-zero if there was any.  Built and run by tests/test_abi.py. */
#include <dlfcn.h>
#include <stdio.h>
#include <string.h>

#include "msa_bank.h"
#include "msa_decode.h"
#include "msa_gather.h"
#include "msa_pool.h"
#include "msa_prefill.h"
#include "msa_route.h"

static int failures = 0;
static void* libs[6];

static void* sym(int lib, const char* name) {
  void* p = dlsym(libs[lib], name);
  if (!p) {
    printf("missing %s\n", name);
    ++failures;
  }
  return p;
}

#define GET(lib, name) __typeof__(name)* p_##name = (__typeof__(name)*)sym(lib, #name)
/* the call returns `want`, and a failing call leaves a message in its library's errfn() */
#define EXPECT(call, want, errfn)                                                                \
  do {                                                                                            \
    msa_status got_ = (call);                                                                     \
    if (got_ != (want)) {                                                                         \
      printf("%s: got %d, want %d\n", #call, (int)got_, (int)(want));                             \
      ++failures;                                                                                 \
    } else if (!(errfn()[0])) {                                                                   \
      printf("%s: no error message\n", #call);                                                    \
      ++failures;                                                                                 \
    }                                                                                             \
  } while (0)
#define EXPECT_OK(call)                                                                          \
  do {                                                                                            \
    msa_status got_ = (call);                                                                     \
    if (got_ != MSA_OK) {                                                                         \
      printf("%s: got %d, want MSA_OK\n", #call, (int)got_);                                      \
      ++failures;                                                                                 \
    }                                                                                             \
  } while (0)

enum { POOL, ROUTE, GATHER, DECODE, PREFILL, BANK };

int main(int argc, char** argv) {
  if (argc != 2) {
    printf("usage: abi_check LIB_DIR\n");
    return 2;
  }
  const char* names[6] = {"pool", "route", "gather", "decode", "prefill", "bank"};
  for (int i = 0; i < 6; ++i) {
    char path[4096];
    snprintf(path, sizeof path, "%s/libmsa_%s.so", argv[1], names[i]);
    libs[i] = dlopen(path, RTLD_NOW | RTLD_LOCAL);
    if (!libs[i]) {
      printf("dlopen %s: %s\n", path, dlerror());
      return 1;
    }
  }
  int32_t dummy[64];
  memset(dummy, 0, sizeof dummy);

  /* pool */
  GET(POOL, msa_count_chunks);
  GET(POOL, msa_pool_blocks);
  GET(POOL, msa_pool_last_error);
  {
    const int64_t tok[4] = {0, 64, 129, 129}; /* 1 + 2 + 0 blocks */
    int64_t out[4] = {-1, -1, -1, -1};
    const int64_t n = p_msa_count_chunks(tok, 3, 64, out);
    if (n != 3 || out[0] != 0 || out[1] != 1 || out[2] != 3 || out[3] != 3) {
      printf("msa_count_chunks: %lld blocks, offsets %lld %lld %lld %lld\n", (long long)n, (long long)out[0],
             (long long)out[1], (long long)out[2], (long long)out[3]);
      ++failures;
    }
    EXPECT(p_msa_pool_blocks(NULL, NULL, NULL, MSA_BF16, NULL, NULL, 3, 3, 8, 128, 64, 1e6f, NULL, NULL, NULL, NULL,
                             NULL, NULL),
           MSA_ERR_INVALID_ARG, p_msa_pool_last_error);
  }

  /* route */
  GET(ROUTE, msa_route_topk_workspace_size);
  GET(ROUTE, msa_route_filter_keys);
  GET(ROUTE, msa_route_topk);
  GET(ROUTE, msa_route_topk_hidden);
  GET(ROUTE, msa_route_wait_selftest);
  GET(ROUTE, msa_route_last_launch_count);
  GET(ROUTE, msa_route_set_profile_events);
  GET(ROUTE, msa_route_set_query_profile_events);
  GET(ROUTE, msa_route_set_pair_mode);
  GET(ROUTE, msa_route_last_error);
  {
    size_t bytes = 0;
    EXPECT_OK(p_msa_route_topk_workspace_size(18, 1, 256, 8, 100000, 1000, 16, &bytes));
    if (bytes == 0) {
      printf("msa_route_topk_workspace_size: 0 bytes\n");
      ++failures;
    }
    EXPECT(p_msa_route_topk_workspace_size(18, 1, 256, 8, 100000, 1000, 65, &bytes), MSA_ERR_INVALID_ARG,
           p_msa_route_last_error);
    EXPECT(p_msa_route_filter_keys(NULL, 1, 1, 8, 128, NULL, NULL), MSA_ERR_INVALID_ARG, p_msa_route_last_error);
    const int32_t qoff[2] = {0, 4};
    EXPECT(p_msa_route_topk(NULL, MSA_F32, qoff, 1, NULL, NULL, NULL, 10, 10, 1, 32, 8, 128, 4, NULL, NULL, NULL, 0,
                            MSA_ROUTE_AUTO, NULL, NULL),
           MSA_ERR_INVALID_ARG, p_msa_route_last_error);
    EXPECT(p_msa_route_topk_hidden(NULL, NULL, 2560, qoff, 1, NULL, NULL, NULL, 10, 10, 1, 32, 8, 128, 4, NULL, NULL,
                                   NULL, 0, MSA_ROUTE_AUTO, NULL, NULL),
           MSA_ERR_INVALID_ARG, p_msa_route_last_error);
    EXPECT(p_msa_route_wait_selftest(1000, 0, NULL, NULL), MSA_ERR_INVALID_ARG, p_msa_route_last_error);
    EXPECT_OK(p_msa_route_set_profile_events(NULL, NULL));
    EXPECT_OK(p_msa_route_set_query_profile_events(NULL, NULL));
    EXPECT_OK(p_msa_route_set_pair_mode(1));
    (void)p_msa_route_last_launch_count();
  }

  /* gather */
  GET(GATHER, msa_gather_kv);
  GET(GATHER, msa_gather_last_error);
  EXPECT(p_msa_gather_kv(NULL, 10, NULL, NULL, 10, NULL, 1, 1, 16, 8, 128, 64, NULL, NULL, NULL, NULL),
         MSA_ERR_INVALID_ARG, p_msa_gather_last_error);

  /* decode */
  GET(DECODE, msa_sparse_decode_workspace_size);
  GET(DECODE, msa_sparse_decode);
  GET(DECODE, msa_sparse_decode_static);
  GET(DECODE, msa_decode_last_error);
  {
    size_t bytes = 0;
    EXPECT_OK(p_msa_sparse_decode_workspace_size(1, 18, 32, 8, &bytes));
    if (bytes != (size_t)18 * 8 * (2080 * 4 + 4) + 4) {
      printf("msa_sparse_decode_workspace_size: %zu bytes\n", bytes);
      ++failures;
    }
    EXPECT(p_msa_sparse_decode_workspace_size(1, 18, 30, 8, &bytes), MSA_ERR_INVALID_ARG, p_msa_decode_last_error);
    EXPECT(p_msa_sparse_decode(NULL, NULL, NULL, 1, 18, 32, 8, 128, NULL, NULL, NULL, 16, NULL, NULL, 64, 16, 1e6f,
                               0.088f, NULL, NULL, 0, NULL, NULL),
           MSA_ERR_INVALID_ARG, p_msa_decode_last_error);
    /* sizes beyond the built-in scratch are refused before any device work */
    EXPECT(p_msa_sparse_decode_static(dummy, dummy, dummy, 64, 512, 32, 8, 128, dummy, dummy, dummy, 4, dummy, dummy,
                                      4, 16, 1e6f, 0.1f, dummy, dummy, NULL),
           MSA_ERR_CAPACITY, p_msa_decode_last_error);
  }

  /* prefill */
  GET(PREFILL, msa_sparse_prefill);
  GET(PREFILL, msa_prefill_last_error);
  EXPECT(p_msa_sparse_prefill(NULL, NULL, NULL, 4, 1, 18, 32, 8, 128, NULL, NULL, NULL, 16, NULL, NULL, 64, 16, 1e6f,
                              0.088f, NULL, NULL, NULL),
         MSA_ERR_INVALID_ARG, p_msa_prefill_last_error);

  /* bank */
  GET(BANK, msa_bank_save);
  GET(BANK, msa_bank_read_info);
  GET(BANK, msa_bank_load);
  GET(BANK, msa_bank_relayout);
  GET(BANK, msa_bank_append_offsets);
  GET(BANK, msa_bank_last_error);
  {
    msa_bank_info info;
    memset(&info, 0, sizeof info);
    EXPECT(p_msa_bank_read_info("/nonexistent/dir/bank.msa", &info), MSA_ERR_IO, p_msa_bank_last_error);
    EXPECT(p_msa_bank_save(NULL, &info, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL), MSA_ERR_INVALID_ARG,
           p_msa_bank_last_error);
    EXPECT(p_msa_bank_load(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL), MSA_ERR_INVALID_ARG,
           p_msa_bank_last_error);
    EXPECT(p_msa_bank_relayout(NULL, NULL, 1, 4, 8, 2048, NULL), MSA_ERR_INVALID_ARG, p_msa_bank_last_error);
    const int64_t old_off[3] = {0, 2, 5}, new_off[3] = {0, 1, 4};
    int64_t out[5] = {0, 0, 0, 0, 0};
    EXPECT_OK(p_msa_bank_append_offsets(old_off, 2, new_off, 2, out));
    if (out[0] != 0 || out[1] != 2 || out[2] != 5 || out[3] != 6 || out[4] != 9) {
      printf("msa_bank_append_offsets: %lld %lld %lld %lld %lld\n", (long long)out[0], (long long)out[1],
             (long long)out[2], (long long)out[3], (long long)out[4]);
      ++failures;
    }
  }

  for (int i = 0; i < 6; ++i) dlclose(libs[i]);
  if (failures) {
    printf("%d failures\n", failures);
    return 1;
  }
  printf("ok\n");
  return 0;
}
