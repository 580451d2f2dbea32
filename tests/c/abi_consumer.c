/* A C99 consumer of the library: it includes the public header, takes the
 * address of every entry point (so the link fails if one is missing) and calls
 * the entry points that need no GPU. */
#include <stdio.h>
#include <string.h>

#include "attn.h"

int main(void) {
  void* entry_points[] = {
      (void*)attn_abi_version,      (void*)attn_status_string,   (void*)attn_fwd,
      (void*)attn_fwd_default_options, (void*)attn_fwd_ex,       (void*)attn_fwd_qk8, (void*)attn_fwd_qkv8,
      (void*)attn_fwd_split,        (void*)attn_fwd_split_qk8,   (void*)attn_fwd_split_count,
      (void*)attn_fwd_split_workspace_size, (void*)attn_bwd_workspace_size, (void*)attn_bwd,
      (void*)attn_bwd_ex,           (void*)attn_bwd_noalloc,     (void*)attn_device_status,
      (void*)attn_set_wait_limit_ns, (void*)attn_exp2_poly_eval, (void*)attn_read_probe};
  for (size_t i = 0; i < sizeof(entry_points) / sizeof(entry_points[0]); ++i)
    if (!entry_points[i]) return 1;
  attn_fwd_options_t opt;
  memset(&opt, 0, sizeof(opt));
  attn_fwd_default_options(&opt);
  if (opt.poly_exp_every != 8 || opt.rescale_threshold != 8.0f) return 2;
  /* argument checks happen before any device work */
  if (attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 2, 2, 8, 8, 64, 0, 0.125f, NULL) != ATTN_ERR_INVALID_ARG) return 3;
  if (attn_bwd_workspace_size(2, 16, 8192, 128) == 0) return 4;
  printf("abi %d, %s\n", attn_abi_version(), attn_status_string(ATTN_ERR_UNSUPPORTED));
  return 0;
}
