// One slice of the paged-decode kernels: element type HILS_DECODE_T (0 = fp32,
// 1 = bf16), head dim HILS_DECODE_D, group size HILS_DECODE_G.  The build compiles
// this file once per slice with those macros set; without them it is empty.
#include "decode_impl.cuh"

#if defined(HILS_DECODE_T) && defined(HILS_DECODE_D) && defined(HILS_DECODE_G)
namespace hils {

#if HILS_DECODE_T
using DecodeElem = __nv_bfloat16;
#else
using DecodeElem = float;
#endif

#define HILS_SLICE_NAME_(t, d, g) run_decode_slice_##t##_##d##_##g
#define HILS_SLICE_NAME(t, d, g) HILS_SLICE_NAME_(t, d, g)

cudaError_t HILS_SLICE_NAME(HILS_DECODE_T, HILS_DECODE_D, HILS_DECODE_G)(const DecodeArgs& a, cudaStream_t st) {
  return launch_decode<DecodeElem, HILS_DECODE_D, HILS_DECODE_G>(a, st);
}

}  // namespace hils
#endif
