// Host-side probe of the UMMA conv's tile planner (no GPU): reads one
// problem per input line and prints the chosen configuration and its
// launch shared memory.  Built and run by tests/test_plan_choice.py.
//
// input:  n c_in c_out h w kt ks rms max_t sm_count e4m3
// output: ok kc nt n_ntiles sub nbuf g_taps pair na nb tmem_cols ctas_per_sm params b_resident
//         xs smem
#include <cstdio>

#include "internal.h"

int main() {
  int n, ci, co, h, w, kt, ks, rms, mt, sms, f8;
  while (std::scanf("%d %d %d %d %d %d %d %d %d %d %d", &n, &ci, &co, &h, &w, &kt, &ks, &rms, &mt,
                    &sms, &f8) == 11) {
    cc3d::UmmaConfig c{};
    const bool ok =
        cc3d::choose_umma_config(n, ci, co, h, w, kt, ks, rms != 0, mt, sms, &c, f8 != 0);
    const size_t smem = ok ? cc3d::umma_launch_smem(c.kc, c.nt, ks, c.na, c.nb, c.tmem_cols,
                                                    c.sub, c.g_taps, c.pair, c.params, c.xs)
                           : 0;
    std::printf("%d %d %d %d %d %d %d %d %d %d %d %d %d %d %d %zu\n", ok ? 1 : 0, c.kc, c.nt,
                c.n_ntiles, c.sub, c.nbuf, c.g_taps, c.pair, c.na, c.nb, c.tmem_cols,
                c.ctas_per_sm, c.params, c.b_resident, c.xs, smem);
  }
  return 0;
}
