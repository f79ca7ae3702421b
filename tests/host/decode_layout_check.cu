// Host-only check of the split decode kernel's shared-memory layout (no GPU):
// for every head dim, query heads per KV head, centroid id width and group
// size, the stage offsets and bulk-copy sizes are multiples of 16 bytes, the
// staged fields fit their regions, the final reduction fits in the stages,
// the zero-point / PSAC k-steps cover their columns, and the CTA's shared
// memory stays within 227 KB for r <= 16 and M <= 512. Compiled and run by
// tests/test_decode_layout.py.
#include <cstdio>
#include <cstdlib>
#include "decode_split.cuh"
using namespace kv2::dsplit;
static int bad = 0;
#define CHECK(c, ...) do { if (!(c)) { printf("FAIL %s: ", #c); printf(__VA_ARGS__); printf("\n"); ++bad; } } while (0)
template <int D, int G, bool U16, int GS>
void check() {
  using C = DCfg<D, G, U16, GS>;
  for (int r : {0, 2, 8, 16, 64, D}) for (int M : {1, 64, 256, 512}) {
    if ((M > 256) != U16 && M > 1) continue;
    CHECK(C::kc_off % 16 == 0 && C::vc_off % 16 == 0 && C::ks_off % 16 == 0 && C::vs_off % 16 == 0 &&
          C::ix_off % 16 == 0 && C::ps_off % 16 == 0, "offsets D%d G%d GS%d", D, G, GS);
    // per-stream copy sizes for a 16-token multiple
    for (int n16 = 16; n16 <= kTile; n16 += 16) {
      CHECK(n16 * C::NW * 4 % 16 == 0 && n16 * C::NG * 4 % 16 == 0 && n16 * C::IDXB % 16 == 0, "copy sizes");
      CHECK((n16 * r * 2) % 16 == 0 || r % 8 != 0, "psac fp16 copy r=%d", r);
    }
    // the staged fields fit their regions
    CHECK(C::vs_off + kTile * C::NG * 4 <= C::ix_off, "vs region");
    CHECK(C::ps_off + kTile * (r + 2) <= C::stage_bytes(r) || r == 0, "int8 psac region r=%d", r);
    CHECK(C::ps_off + kTile * r * 2 <= C::stage_bytes(r), "psac region");
    CHECK(C::stage_bytes(r) % 16 == 0, "stage size");
    CHECK(C::stages_bytes(r) >= C::red_bytes, "reduction fits");
    const size_t total = split_smem<D, G, U16, GS>(M, r);
    if (r <= 16) CHECK(total <= 227 * 1024, "smem %zu D%d G%d U16%d GS%d M%d r%d", total, D, G, U16, GS, M, r);
    CHECK(C::xk(r) * 16 >= C::NGP + r, "aux k-steps");
    CHECK(C::NGP % 2 == 0 && C::NGP >= C::NG, "NGP");
    CHECK(C::MTV <= C::WPG, "p.v group per warp");
    CHECK(C::lg_bytes + C::wt_bytes >= (G * D) * 4 + 4, "prologue scratch");
  }
  printf("D%3d G%d U16 %d GS%3d: NG %d NGP %d XK(8) %d stage %d B, smem(M=%d,r=16) %zu B\n", D, G, int(U16), GS,
         C::NG, C::NGP, C::xk(8), C::stage_bytes(16), U16 ? 512 : 256, split_smem<D, G, U16, GS>(U16 ? 512 : 256, 16));
}
template <int D, bool U16, int GS> void all_g() { check<D, 1, U16, GS>(); check<D, 2, U16, GS>(); check<D, 4, U16, GS>(); check<D, 8, U16, GS>(); }
int main() {
  all_g<64, false, 32>(); all_g<64, true, 32>(); all_g<64, false, 64>(); all_g<64, true, 64>();
  all_g<128, false, 32>(); all_g<128, true, 32>(); all_g<128, false, 64>(); all_g<128, true, 64>();
  all_g<128, false, 128>(); all_g<128, true, 128>();
  printf(bad ? "%d FAILURES\n" : "all layout checks passed\n", bad);
  return bad != 0;
}
