#include "common.cuh"
namespace pararnn {
int launch_lstm_fwd(const CUtensorMap&, bool, const FwdParams&, int, cudaStream_t) { return 1; }
int lstm_chunk_steps() { return 128; }
int lstm_max_cluster(bool) { return 8; }
int adjoint_chunk_steps(int) { return 256; }
size_t adjoint_ws_bytes(int, int, int, int) { return 256; }
int launch_adjoint(int, bool, const CUtensorMap&, const void*, const float*, const float*, const float*, const float*, const float*, const float*, const float*, float*, float*, float*, float*, float*, int, int, int, int*, void*, cudaStream_t) { return 1; }
}
