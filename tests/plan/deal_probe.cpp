// Host-side probe of the per-call layer choice (no GPU): for one problem per
// input line, the relative cost of a call on the plan's tiles (chosen for
// max_t) and on the tiles chosen for one frame.  Built and run by
// tests/test_plan_choice.py.
//
// input:  n c_in c_out h w kt ks rms max_t sm_count t_out cached stride_t
// output: ok cost_plan cost_one_frame pair_plan pair_one_frame
#include <cstdio>

#include "internal.h"

int main() {
  int n, ci, co, h, w, kt, ks, rms, mt, sms, to, cached, st;
  while (std::scanf("%d %d %d %d %d %d %d %d %d %d %d %d %d", &n, &ci, &co, &h, &w, &kt, &ks,
                    &rms, &mt, &sms, &to, &cached, &st) == 13) {
    cc3d::UmmaConfig c{}, c1{};
    const bool ok = cc3d::choose_umma_config(n, ci, co, h, w, kt, ks, rms != 0, mt, sms, &c) &&
                    cc3d::choose_umma_config(n, ci, co, h, w, kt, ks, rms != 0, 1, sms, &c1);
    const long long a = ok ? cc3d::umma_deal_cost(c, n, to, h, w, kt, st, cached != 0, sms) : 0;
    const long long b = ok ? cc3d::umma_deal_cost(c1, n, to, h, w, kt, st, cached != 0, sms) : 0;
    std::printf("%d %lld %lld %d %d\n", ok ? 1 : 0, a, b, c.pair, c1.pair);
  }
  return 0;
}
