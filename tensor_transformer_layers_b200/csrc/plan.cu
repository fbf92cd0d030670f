// plan.cu - host-side choice of the GEMM tiling for one launch (no device code).
//
// gemm.cu has three tilings of the same output-stationary GEMM: CTA pairs with
// 256 x 256 tiles (256 x 128 output columns in SwiGLU mode), and one CTA per
// 128 x 256 or 128 x 128 tile.  Each CTA (or pair) walks its tiles with the
// whole K loop, so a launch takes ceil(tiles / slots) rounds of tiles.  The
// plan compares the per-SM work of those rounds: a pair tile is two 128 x 128
// blocks per SM, a 128 x 256 tile two, a 128 x 128 tile one, and a 128 x 128
// block costs about 1.5x as much on its own (the MMA re-reads A from shared
// memory for every 128 columns instead of 256).
#include "internal.h"

namespace tp {

int gemm_tile_plan(int64_t M, int64_t N, int groups, bool swiglu, int num_sms) {
  if (M <= 0 || N <= 0 || groups <= 0 || num_sms <= 0) return kPlanCta128x256;
  auto rounds = [](int64_t tiles, int64_t slots) { return (tiles + slots - 1) / slots; };
  const int64_t m128 = (M + 127) / 128;
  const int64_t t128 = m128 * ((N + 127) / 128) * groups;
  if (M >= 256) {
    if (swiglu) return kPlanPair;
    const int64_t pair_tiles = ((M + 255) / 256) * ((N + 255) / 256) * groups;
    return 3 * rounds(t128, num_sms) < 4 * rounds(pair_tiles, gemm_max_active_pairs(num_sms)) ? kPlanCta128x128
                                                                                                  : kPlanPair;
  }
  if (swiglu) return kPlanCta128x256;
  const int64_t t256 = m128 * ((N + 255) / 256) * groups;
  return 3 * rounds(t128, num_sms) < 4 * rounds(t256, num_sms) ? kPlanCta128x128 : kPlanCta128x256;
}

}  // namespace tp
