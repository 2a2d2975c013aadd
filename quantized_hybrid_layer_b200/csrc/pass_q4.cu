// Instantiation of the persistent layer-stage pass for Q4_0 weights (NT = 1..4).
#include "launch.h"

namespace qhl {
template struct PassOps<kQ4_0>;
}  // namespace qhl
