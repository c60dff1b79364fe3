// Associative (gradient-ascent, weight-norm-free) linear-attention mode.
#include "internal.h"

namespace ttt {
size_t assoc_workspace_bytes(int, int, int, int, int) { return 0; }
bool assoc_supported(int, int, int) { return false; }
int launch_assoc(const StateArgs&, const LaunchCtx& ctx) {
  *ctx.msg = "ttt_assoc_scan_fwd: not built yet";
  return kUnsupported;
}
}  // namespace ttt
