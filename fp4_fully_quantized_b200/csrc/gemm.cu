// gemm.cu -- kernel behind fp4_gemm.
//
// The product is the one of the "FP4" page (How it works): E2M1 operands with
// per-block scales on the tensor cores, FP32 accumulation.  gemm_sfst.cu runs
// it with one SM per 128 x 256 output tile (persistent CTAs, tcgen05 MMAs
// with operands staged by TMA and scale factors staged by tcgen05.st).
#include "internal.h"

namespace fp4impl {

fp4_status gemm_launch(const GemmArgs& g, cudaStream_t s) {
  return gemm_launch_sfst(g, s);
}

}  // namespace fp4impl
