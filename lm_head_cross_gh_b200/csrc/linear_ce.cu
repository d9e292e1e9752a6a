// Chunked fused linear cross-entropy (placeholder until the tcgen05 GEMMs land).
#include "linear_ce.h"

namespace gh {

gh_status_t linear_ce_run(const LinearCeArgs&, cudaStream_t) { return GH_ERR_UNSUPPORTED; }

}  // namespace gh
