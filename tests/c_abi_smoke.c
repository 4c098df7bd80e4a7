/* Calls libhs2 through its C header from plain C (no CUDA headers, no GPU):
 * size queries and argument checks only, none of which launch anything.
 * Prints one "name value" line per check for tests/test_c_abi.py. */
#include <stdio.h>
#include <string.h>

#include "hs2.h"

int main(void) {
  hs2_shape s;
  memset(&s, 0, sizeof s);
  s.L = 131072;
  s.Hq = 64;
  s.Hkv = 8;
  s.d = 128;
  s.block = 64;
  s.topk = 1024;
  s.recent = 128;
  s.kv_dtype = HS2_KV_BF16;
  s.q_tok_stride = 64 * 128;
  s.q_head_stride = 128;
  s.kv_tok_stride = 8 * 128;
  s.kv_head_stride = 128;

  size_t ws = 0;
  int rc = hs2_full_attn_select(&s, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, &ws, NULL, 0, 0, NULL);
  printf("full_ws_rc %d\nfull_ws_bytes %zu\n", rc, ws);

  size_t fa_ws = 123;
  rc = hs2_attn_fwd_ws(&s, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, &fa_ws, NULL);
  printf("fa_ws_rc %d\nfa_ws_bytes_bf16 %zu\n", rc, fa_ws);

  s.kv_dtype = HS2_KV_E4M3;
  rc = hs2_attn_fwd_ws(&s, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, &fa_ws, NULL);
  printf("fa_ws_bytes_e4m3 %zu\n", fa_ws);
  s.kv_dtype = HS2_KV_BF16;

  size_t dec_ws = 0;
  rc = hs2_sparse_decode_workspace(&s, 1, &dec_ws);
  printf("decode_ws_rc %d\ndecode_ws_bytes %zu\n", rc, dec_ws);

  s.d = 64; /* unsupported head size: refused before any launch */
  rc = hs2_full_attn_select(&s, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, &ws, NULL, 0, 0, NULL);
  printf("bad_d_rc %d\n", rc);

  printf("version %d\n", hs2_version());
  printf("strerror_timeout %s\n", hs2_strerror(HS2_ERR_TIMEOUT));
  return 0;
}
