// Placeholder until the tcgen05 kernel lands: reports the shape as unsupported.
#include "mla_tc.h"

namespace mla {
bool tc_supported(int, int, int, int, int, int, int) { return false; }
int tc_auto_workers(int sms, int) { return sms / 2; }
bool tc_workers_ok(int, int) { return false; }
cudaError_t launch_tc_decode(const DecodeArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace mla
