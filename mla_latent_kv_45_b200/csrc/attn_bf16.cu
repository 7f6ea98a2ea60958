// bf16 latent attention (DeepSeek-V2 sizes).
#include "sm100.h"

namespace mla {
namespace sm100 {

cudaError_t launch_attn(const AttnArgs &a, int parts, cudaStream_t s) {
  return launch_attn_simt<__nv_bfloat16>(a, parts, s);
}

}  // namespace sm100
}  // namespace mla
