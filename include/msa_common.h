/* Common types of the MSA (Memory Sparse Attention) hot-path libraries.
 *
 * One shared library per step of the online/offline path described on the MSA pages
 * ("MSA端到端可训练记忆模型完整开源，支持亿级Token上下文", sections 架构 and 推理流水线), plus
 * the query's prefill and bank persistence:
 *   libmsa_pool.so    offline block compression        (msa_pool.h)
 *   libmsa_route.so   routing scores + top-k documents (msa_route.h)
 *   libmsa_gather.so  host -> device load of selection (msa_gather.h)
 *   libmsa_decode.so  sparse decode attention          (msa_decode.h)
 *   libmsa_prefill.so the query's own tokens through sparse attention (msa_prefill.h)
 *   libmsa_bank.so    bank file save / load, append re-layout (msa_bank.h)
 *
 * Conventions shared by every entry point:
 *  - Every call returns an msa_status; nothing else crosses the ABI on failure.  The
 *    library's msa_<lib>_last_error() returns a thread-local message for the last
 *    failing call of that library on this thread.
 *  - Every buffer is owned by the caller.  The libraries never allocate device or
 *    host memory (the one exception, msa_sparse_decode_static, holds a fixed array of
 *    its own); calls that need scratch space take a caller buffer whose size comes
 *    from a *_workspace_size query or is stated in the header.
 *  - Calls are asynchronous on the stream they are given (NULL = legacy default
 *    stream).  Host-side argument checks happen before anything is enqueued.
 *  - Conditions only the GPU can see (capacity overflow, a bad document id, a full
 *    local cache) OR a bit into the caller's int32 device word dev_err; read it after
 *    synchronising.  The kernels never trap.
 *  - Only sm_100 devices (B200) are supported; other devices get MSA_ERR_UNSUPPORTED.
 */
#ifndef MSA_COMMON_H
#define MSA_COMMON_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum msa_status {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1, /* null pointer, bad size, unsupported combination of sizes */
  MSA_ERR_UNSUPPORTED = 2, /* device is not sm_100, or a dtype the call does not take */
  MSA_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  MSA_ERR_CAPACITY = 4,    /* a caller buffer is too small (workspace, cache) */
  MSA_ERR_TIMEOUT = 5,     /* reserved for host waits with a time limit */
  MSA_ERR_IO = 6           /* a bank file cannot be opened, read or written, or fails its checks */
} msa_status;

typedef enum msa_dtype { MSA_F32 = 0, MSA_BF16 = 1 } msa_dtype;

/* Same object as cudaStream_t; declared here so the headers need no CUDA include. */
typedef struct CUstream_st* msa_stream_t;

/* Bits OR-ed into *dev_err by the kernels. */
#define MSA_DEVERR_CAPACITY 1u    /* a selection does not fit max_mem_chunks (clamped)   */
#define MSA_DEVERR_BAD_DOC 2u     /* a document id outside [0, n_docs) (skipped)         */
#define MSA_DEVERR_LOCAL_FULL 4u  /* local cache has no room for the new token (skipped) */
#define MSA_DEVERR_BAD_OFFSETS 8u /* offsets disagree with the declared counts           */
#define MSA_DEVERR_TIMEOUT 16u    /* a bounded in-kernel wait ran out (work abandoned)    */
#define MSA_DEVERR_UNCERTIFIED 32u /* tensor-core routing: a selection whose certification
                                      failed with no further stage to send it to (kept in
                                      the ABI; the routing's last stage is an exact scan,
                                      so msa_route_topk does not raise it) */

/* Bytes of one memory block of one layer in a bf16 bank:
 * routing key H*d*2; content key + value 2*H*d*2. */
#define MSA_ROUTER_BYTES_PER_BLOCK(H, d) ((size_t)(H) * (size_t)(d) * 2u)
#define MSA_CONTENT_BYTES_PER_BLOCK(H, d) ((size_t)(H) * (size_t)(d) * 4u)

#ifdef __cplusplus
}
#endif

#endif /* MSA_COMMON_H */
