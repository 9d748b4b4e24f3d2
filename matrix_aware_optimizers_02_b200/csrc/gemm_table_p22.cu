// Table-mode GEMM kernels with 2 plane(s) of A and 2 plane(s) of B.
#include "gemm_table.cuh"

namespace mao {
template mao_status launch_table_planes<2, 2>(const GemmTableParams&, int, int, cudaStream_t, int, double, bool);
}  // namespace mao
