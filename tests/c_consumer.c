/*
 * A plain C99 consumer of the library: it includes only include/diffattn.h,
 * links libdiffattn.so, and checks the host-side contract that holds without
 * a GPU -- argument validation returns its documented code before any CUDA
 * call, workspace sizes follow their formulas, N = 0 is a no-op, and every
 * entry point has the signature the header declares (taking each address
 * into a pointer of the declared type fails to compile otherwise).
 * Built and run by tests/test_c_consumer.py; prints one line per failed
 * check and exits with the number of failures.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "diffattn.h"

static int failures = 0;

#define EXPECT_EQ(got, want)                                                         \
  do {                                                                               \
    long long g_ = (long long)(got), w_ = (long long)(want);                         \
    if (g_ != w_) {                                                                  \
      printf("line %d: %s = %lld, expected %lld\n", __LINE__, #got, g_, w_);         \
      ++failures;                                                                    \
    }                                                                                \
  } while (0)

int main(void) {
  /* a 4096-aligned address that is never dereferenced: validation rejects the
     call before any use of it */
  void* fake = (void*)(uintptr_t)4096;
  void* fake16 = (void*)(uintptr_t)(4096 + 16); /* 16- but not 32-byte aligned */
  float* ff = (float*)fake;
  const cudaStream_t s0 = 0;

  /* the declared signatures */
  int (*p_fwd)(const void*, const void*, const void*, void*, int, int, int, int, int, int, const float*, float,
               const float*, float, cudaStream_t) = diffattn_fwd;
  int (*p_q4)(const void*, int, int, int, int, void*, float*, cudaStream_t) = diffattn_quantize_qk4;
  size_t (*p_ws)(int, int, int, int) = diffattn_bwd_workspace_size;
  const char* (*p_str)(int) = diffattn_status_string;
  (void)p_fwd;
  (void)p_q4;
  (void)p_ws;

  EXPECT_EQ(diffattn_version() >= 101, 1);
  EXPECT_EQ(strcmp(p_str(DIFFATTN_OK), "ok"), 0);
  EXPECT_EQ(strcmp(diffattn_status_string(DIFFATTN_ERR_INVALID_ARG), "invalid argument"), 0);
  EXPECT_EQ(diffattn_set_wait_limit_ns(-1), DIFFATTN_ERR_INVALID_ARG);
  EXPECT_EQ(diffattn_set_wait_limit_ns(0), DIFFATTN_OK); /* restores the default */
  EXPECT_EQ(diffattn_device_status(NULL), DIFFATTN_ERR_INVALID_ARG);

  /* lambda */
  EXPECT_EQ(diffattn_lambda(NULL, ff, ff, ff, 8, 0.5f, ff, s0), DIFFATTN_ERR_INVALID_ARG);

  /* prefill */
  EXPECT_EQ(diffattn_fwd(NULL, fake, fake, fake, DIFFATTN_BF16, 1, 16, 2, 128, 1, ff, 0.5f, ff, 1e-5f, s0),
            DIFFATTN_ERR_INVALID_ARG);
  EXPECT_EQ(diffattn_fwd(fake, fake, fake, fake, 7, 1, 16, 2, 128, 1, ff, 0.5f, ff, 1e-5f, s0),
            DIFFATTN_ERR_INVALID_ARG);
  EXPECT_EQ(diffattn_fwd(NULL, NULL, NULL, NULL, DIFFATTN_BF16, 1, 0, 2, 128, 1, NULL, 0.5f, NULL, 1e-5f, s0),
            DIFFATTN_OK); /* N = 0 */
  EXPECT_EQ(diffattn_fwd_mode(fake, fake, fake, fake, DIFFATTN_BF16, 1, 16, 2, 128, 1, ff, 0.5f, ff, 1e-5f, 3, s0),
            DIFFATTN_ERR_INVALID_ARG);

  /* low-bit queries and keys */
  EXPECT_EQ(diffattn_quantize_qk(fake, 1, 16, 2, 12, fake, ff, s0), DIFFATTN_ERR_INVALID_ARG); /* d % 8 */
  EXPECT_EQ(diffattn_quantize_qk4(NULL, 1, 16, 2, 128, fake, ff, s0), DIFFATTN_ERR_INVALID_ARG);
  EXPECT_EQ(diffattn_fwd_qk8(fake, ff, fake, ff, fake, fake, 1, 16, 2, 64, 1, ff, 0.5f, ff, 1e-5f, 0, s0),
            DIFFATTN_ERR_UNSUPPORTED);
  EXPECT_EQ(diffattn_fwd_qk4(fake, ff, fake, ff, fake, fake, 1, 16, 2, 64, 1, ff, 0.5f, ff, 1e-5f, 0, s0),
            DIFFATTN_ERR_UNSUPPORTED);
  EXPECT_EQ(diffattn_fwd_qk4(fake16, ff, fake, ff, fake, fake, 1, 16, 2, 128, 1, ff, 0.5f, ff, 1e-5f, 0, s0),
            DIFFATTN_ERR_INVALID_ARG);

  /* backward */
  EXPECT_EQ(diffattn_bwd_workspace_size(1, 16, 2, 64), 4 * 16 * 2 * 128 + 16 * 16 * 2);
  EXPECT_EQ(diffattn_bwd_workspace_size(0, 16, 2, 64), 0);
  EXPECT_EQ(diffattn_bwd(fake, fake, fake, fake, DIFFATTN_F32, 1, 16, 2, 64, 1, ff, 0.5f, ff, 1e-5f, 0, ff, ff, ff,
                         ff, ff, NULL, (size_t)1 << 30, s0),
            DIFFATTN_ERR_WORKSPACE);
  EXPECT_EQ(diffattn_bwd_tc_workspace_size(0, 16, 2, 128), 0);

  /* decode */
  EXPECT_EQ(diffattn_decode_workspace_size(0, 12, 128, 4096), 0);
  EXPECT_EQ(diffattn_decode_workspace_size(4, 12, 128, 4096) > 0, 1);

  /* projections */
  EXPECT_EQ(diffattn_rope_table(16, 7, 10000.0, ff, s0), DIFFATTN_ERR_INVALID_ARG); /* odd d */

  if (failures == 0) printf("c consumer ok\n");
  return failures;
}
