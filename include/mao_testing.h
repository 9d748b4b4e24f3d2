/*
 * mao_testing.h — entry points of libmao that exist for verification: they
 * expose the grouped tensor-core GEMM core on its own so that tests can check
 * it against a plain fp32 matrix product, independently of any optimizer.
 * Same conventions as mao.h (caller-owned device buffers, 16-byte alignment,
 * validation before any launch, no synchronisation).
 */
#ifndef MAO_TESTING_H_
#define MAO_TESTING_H_

#include "mao.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MAO_GEMM_BF16 = 0,
  MAO_GEMM_SPLIT3 = 1,
  MAO_GEMM_BF16_FOLD = 2,
  MAO_GEMM_SPLIT3_BF16 = 3,
  MAO_GEMM_BF16_SPLIT3 = 4,
  MAO_GEMM_SPLIT2 = 5
} mao_gemm_kind;

/* Flags OR-ed into a kind: run the problems on the one-CTA kernel (128 x 128
 * tiles; 128 x 256 for bf16 operands) or on the CTA-pair kernel (256 x 128 tiles
 * for the fp32-faithful kinds, 256 x 256 for MAO_GEMM_BF16; tcgen05 cta_group::2);
 * without a flag the library chooses as it does inside the optimizer steps (the
 * pair kernel for products with a three-plane operand, and for the bf16
 * Newton-Schulz products, whose 256-row tiles fill the GPU). */
#define MAO_GEMM_FORCE_ONE_CTA 16
#define MAO_GEMM_FORCE_CTA_PAIR 32

/*
 * D[b] = A[b] * B[b]^T for b < batch, with fp32 accumulation and fp32 D.
 *   kind MAO_GEMM_BF16:   A, B bf16; one bf16 tensor-core product, accumulated
 *                         over the whole K in the tensor memory (the Newton-Schulz
 *                         kernels' core).
 *   kind MAO_GEMM_SPLIT3: A, B fp32; each split into three bf16 planes
 *                         x = x0 + x1 + x2 and the six significant cross
 *                         products accumulated in fp32 (fp32-faithful).
 *   kind MAO_GEMM_BF16_FOLD:   A, B bf16; the exact bf16 product with partial
 *                         sums over 256 of K folded in fp32 registers (the
 *                         SOAP/FOAM factor products of a bf16 gradient).
 *   kind MAO_GEMM_SPLIT3_BF16: A fp32 (three planes), B bf16 (one plane): three
 *                         products, fp32-faithful.
 *   kind MAO_GEMM_BF16_SPLIT3: A bf16, B fp32: the mirror of the previous kind.
 *   kind MAO_GEMM_SPLIT2: A, B fp32 held as two bf16 planes each, products
 *                         x0 y0 + x0 y1 + x1 y0 (about 16 significant bits).
 * Layouts (row-major, contiguous batches):
 *   a_mn_major = 0: A is [batch][M][K]; 1: A is [batch][K][M]
 *   b_mn_major = 0: B is [batch][N][K]; 1: B is [batch][K][N]
 *   D is [batch][M][N].
 * The innermost extent of A and B must be a multiple of 8 elements, N a
 * multiple of 4.  workspace: >= mao_test_gemm_workspace_size() bytes, 256-byte
 * aligned (holds the device status word and, for SPLIT3, the split operands and
 * the problem descriptors).
 */
/*
 * Kernel choice for every tensor-core product of this process (table-mode and
 * the bf16 Newton-Schulz products; verification of the optimizer steps on each
 * kernel): 0 = the library's choice (default), 1 = the one-CTA kernel always,
 * 2 = the CTA-pair kernel always, whatever the launch's size or plane counts.
 * Affects only calls made after it returns; not thread-safe with concurrent steps.
 */
MAO_API mao_status mao_test_set_table_kernel(int32_t policy);

/*
 * Failure-path check of the bounded device waits: one thread waits, through the
 * library's bounded mbarrier wait, on a barrier phase that nothing completes.  After
 * the wait limit (1 s of %globaltimer) it records MAO_ERR_TIMEOUT with site 40 in the
 * status word at workspace offset 0 and the kernel returns; the context stays usable.
 * Read the result with mao_workspace_status.  workspace: >= 16 bytes, 256-byte
 * aligned (its status word is cleared first).  No synchronisation.
 */
MAO_API mao_status mao_test_wait_timeout(void* workspace, size_t ws_bytes, mao_stream_t stream);

MAO_API mao_status mao_test_gemm_workspace_size(int32_t kind, int32_t batch, int32_t M, int32_t N, int32_t K,
                                        size_t* bytes);
MAO_API mao_status mao_test_gemm(int32_t kind, int32_t a_mn_major, int32_t b_mn_major, const void* A, const void* B,
                         float* D, int32_t batch, int32_t M, int32_t N, int32_t K, void* workspace,
                         size_t ws_bytes, mao_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MAO_TESTING_H_ */
