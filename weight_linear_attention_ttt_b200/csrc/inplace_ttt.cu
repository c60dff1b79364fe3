// In-Place TTT W_down chunk update.
#include "internal.h"

namespace ttt {
size_t inplace_workspace_bytes(int, int, int, int) { return 0; }
bool inplace_supported(int, int, int, int, std::string* why) {
  *why = "not built yet";
  return false;
}
int launch_inplace(const InplaceArgs&, const LaunchCtx& ctx) {
  *ctx.msg = "inplace_ttt_chunk_fwd: not built yet";
  return kUnsupported;
}
}  // namespace ttt
