// Launcher of the row-layout decode kernel (attend_rows.cuh) for contiguous caches; paged pools go to the
// instances of attend_rows_paged.cu.
#include "attend_rows_dispatch.cuh"

namespace axr {

axr_status attend_rows_paged_launch(int d, int bits, int G, bool vq, const DecodeArgs& a, cudaStream_t st);

axr_status attend_rows_launch(int d, int bits, int G, bool vq, const DecodeArgs& a, cudaStream_t st) {
  if (a.block_table) return attend_rows_paged_launch(d, bits, G, vq, a, st);
  return rows_detail::dispatch<false>(d, bits, G, vq, a, st);
}

}  // namespace axr
