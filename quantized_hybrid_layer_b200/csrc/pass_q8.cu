// Instantiation of the persistent layer-stage pass for Q8_0 weights (NT = 1..4).
#include "launch.h"

namespace qhl {
template struct PassOps<kQ8_0>;
}  // namespace qhl
