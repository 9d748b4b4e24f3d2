// Table-mode GEMM kernels with 1 plane(s) of A and 1 plane(s) of B.
#include "gemm_table.cuh"

namespace mao {
template mao_status launch_table_planes<1, 1>(const GemmTableParams&, int, int, cudaStream_t, int, double, bool);
}  // namespace mao
