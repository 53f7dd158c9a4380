// Tensor-core (tcgen05 / TMEM / TMA) LLA decode attention.  Placeholder until
// the kernel lands: reports every shape as unsupported.
#include "lla_internal.cuh"

bool lla_tc_supported(const lla_codec*) { return false; }
size_t lla_tc_workspace_bytes(const lla_codec*, int, int) { return 0; }
lla_status lla_decode_tc(const lla_decode_call&, int) { return LLA_ERR_UNSUPPORTED_SHAPE; }
lla_status lla_build_phi_tiles(lla_codec*, cudaStream_t) { return LLA_OK; }
