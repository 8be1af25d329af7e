// K3: placeholder translation unit for the tcgen05 kernel.
#include "plsh_internal.h"

namespace plsh {
int launch_attention_tc(const AttnArgs& a, cudaStream_t st) { return launch_attention_simt(a, st); }
}  // namespace plsh
