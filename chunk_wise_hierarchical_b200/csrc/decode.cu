// Paged decode dispatch.  The kernels live in decode_impl.cuh; each (element type,
// head dim, group size) slice of them is compiled from decode_slice.cu as its own
// object, so the slices build in parallel.
#include "decode_impl.cuh"

namespace hils {

// Ranges per sequence: ranges of kMinRange..kMaxRange chunks, enough of them for about
// kScanCtasTarget CTAs over the batch.  A pure function of the shape, so the workspace
// layout and the launch agree.
int decode_splits(int batch, int max_chunks) {
  const int lo = (max_chunks + kMaxRange - 1) / kMaxRange;
  const int hi = max(1, (max_chunks + kMinRange - 1) / kMinRange);
  const int want = (kScanCtasTarget + max(1, batch) - 1) / max(1, batch);
  return max(lo, min(hi, want));
}
bool decode_supported(int h, int d) { return h * d <= 8 * kScanThreads * 4; }
bool decode_merge_supported(int batch, int max_chunks, int top_k) {
  return decode_merge_fits(decode_splits(batch, max_chunks), top_k);
}

#define HILS_DECLARE_SLICE(t, d, g) \
  cudaError_t run_decode_slice_##t##_##d##_##g(const DecodeArgs& a, cudaStream_t st);
#define HILS_DECLARE_GROUPS(t, d) \
  HILS_DECLARE_SLICE(t, d, 1) HILS_DECLARE_SLICE(t, d, 2) HILS_DECLARE_SLICE(t, d, 4) HILS_DECLARE_SLICE(t, d, 8)
HILS_DECLARE_GROUPS(0, 64)
HILS_DECLARE_GROUPS(0, 128)
HILS_DECLARE_GROUPS(1, 64)
HILS_DECLARE_GROUPS(1, 128)

using DecodeSlice = cudaError_t (*)(const DecodeArgs&, cudaStream_t);
#define HILS_GROUPS(t, d) \
  { run_decode_slice_##t##_##d##_1, run_decode_slice_##t##_##d##_2, \
    run_decode_slice_##t##_##d##_4, run_decode_slice_##t##_##d##_8 }
// [bf16][d == 128][log2 of the group size]
static const DecodeSlice kSlices[2][2][4] = {
    {HILS_GROUPS(0, 64), HILS_GROUPS(0, 128)},
    {HILS_GROUPS(1, 64), HILS_GROUPS(1, 128)},
};

cudaError_t run_decode(DecodeArgs a, cudaStream_t st) {
  a.nsplit = decode_splits(a.b, a.max_chunks);
  a.range = (a.max_chunks + a.nsplit - 1) / a.nsplit;
  int lg;
  switch (a.h / a.g) {
    case 1: lg = 0; break;
    case 2: lg = 1; break;
    case 4: lg = 2; break;
    case 8: lg = 3; break;
    default: return cudaErrorInvalidValue;
  }
  return kSlices[a.bf16 ? 1 : 0][a.d == 64 ? 0 : 1][lg](a, st);
}

}  // namespace hils
