// The row-layout decode kernel (attend_rows.cuh) instantiated for paged pools: rows through the block table.
#include "attend_rows_dispatch.cuh"

namespace axr {

axr_status attend_rows_paged_launch(int d, int bits, int G, bool vq, const DecodeArgs& a, cudaStream_t st) {
  return rows_detail::dispatch<true>(d, bits, G, vq, a, st);
}

}  // namespace axr
