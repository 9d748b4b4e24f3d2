// Table-mode GEMM kernels with 3 plane(s) of A and 1 plane(s) of B.
#include "gemm_table.cuh"

namespace mao {
template mao_status launch_table_planes<3, 1>(const GemmTableParams&, int, int, cudaStream_t, int, double, bool);
}  // namespace mao
