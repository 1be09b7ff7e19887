// Order-1 tensor-core (tcgen05/TMEM, TMA) path of the SSD forward operator.
#include "ssd_internal.h"

namespace ssd {

bool tc_order1_supports(int, int, int, int, int, int) { return false; }
size_t tc_order1_workspace(int, int, int, int, int) { return 0; }
int launch_tc_order1(const FwdArgs &, const Plan &) { return SSD_ERR_UNSUPPORTED; }

}  // namespace ssd
