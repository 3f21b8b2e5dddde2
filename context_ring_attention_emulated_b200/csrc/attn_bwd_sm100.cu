// attn_bwd_sm100.cu -- placeholder until the tensor-core backward lands.
#include "internal.h"

namespace rattn {
rattn_status launch_bwd_sm100(const BwdArgs&, const DevCtx&) { return RATTN_ERR_UNSUPPORTED; }
}  // namespace rattn
