// decode_step.cu -- one decode step of block top-k sparse attention in one call.
//
// Kinetics (block top-k section): at every step the block representation is
// kept current, every block is scored against the query, the K' best blocks
// are kept, and attention runs over their tokens only.  ksa_decode_step issues
// the step's launches -- the fused selection (last-block refresh + scoring,
// then ranking) and the attention over its block lists -- from one call, on
// one workspace, so a serving loop crosses the library boundary once per step.
// The results are those of the two calls, bit for bit: the same launches.
//
// (A one-launch form -- a cooperative persistent kernel with the three phases
// separated by a grid barrier and per-row flags -- was built and measured: it
// was slower than these launches on every workload, see the design notes.)
#include "ksa_internal.h"

namespace ksa {

size_t decode_step_workspace_bytes(int B, int Hq, int Hkv, int D, int T, int bs, int num_sms) {
  return select_workspace_bytes(B, Hkv, T, bs) + attn_workspace_bytes(B, Hq, Hkv, D, num_sms);
}

cudaError_t launch_decode_step(const SelectArgs &sa, const uint16_t *K, const AttnArgs &aa,
                               void *ws, int num_sms, cudaStream_t stream) {
  const size_t sel_bytes = select_workspace_bytes(sa.B, sa.Hkv, sa.T, sa.bs);
  cudaError_t err = launch_select_blocks(sa, K, ws, num_sms, stream);
  if (err != cudaSuccess) return err;
  return launch_sparse_decode_attn(aa, static_cast<uint8_t *>(ws) + sel_bytes, num_sms, stream);
}

}  // namespace ksa
