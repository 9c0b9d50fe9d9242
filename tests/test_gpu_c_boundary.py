"""The C boundary on the GPU, called from C (marked gpu).

A strict C99 program that knows nothing but include/llama_attn.h and the CUDA
runtime API allocates device memory with cudaMalloc, copies in seeded inputs
written here, and calls llama_rope_table, llama_attn_prefill (with the
workspace llama_attn_prefill_workspace_bytes asks for) and llama_attn_decode
on small GQA problems, all on the legacy default stream.  It writes the
outputs to files; they are compared here with the fp64 oracle at the bf16
tolerance of the other parity tests, and the prefill output shape is the
[b, S, H*D] head concatenation of "[HuggingFace Transformers] LlamaAttention
source walkthrough", section 2 step 6.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
from llama_gqa_causal_b200 import api, build, workloads as W

pytestmark = pytest.mark.gpu

CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")

PROGRAM = r"""
#include <stdio.h>
#include <stdlib.h>
#include <cuda_runtime_api.h>
#include "llama_attn.h"

#define CK(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) { \
  fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_)); return 2; } } while (0)
#define LA(x) do { int s_ = (x); if (s_ != LLAMA_OK) { \
  fprintf(stderr, "%s: %s\n", #x, llama_attn_status_string(s_)); return 3; } } while (0)

static char dir[4096];

static const char* path(const char* name) {
  static char buf[4200];
  snprintf(buf, sizeof buf, "%s/%s", dir, name);
  return buf;
}

/* read a whole input file into fresh device memory of exactly `bytes` */
static int upload(const char* name, size_t bytes, void** dev) {
  FILE* f = fopen(path(name), "rb");
  void* host = malloc(bytes);
  size_t got;
  if (!f || !host) return 4;
  got = fread(host, 1, bytes, f);
  fclose(f);
  if (got != bytes) return 5;
  CK(cudaMalloc(dev, bytes));
  CK(cudaMemcpy(*dev, host, bytes, cudaMemcpyHostToDevice));
  free(host);
  return 0;
}

static int download(const char* name, const void* dev, size_t bytes) {
  void* host = malloc(bytes);
  FILE* f;
  if (!host) return 4;
  CK(cudaMemcpy(host, dev, bytes, cudaMemcpyDeviceToHost));
  f = fopen(path(name), "wb");
  if (!f || fwrite(host, 1, bytes, f) != bytes) return 6;
  fclose(f);
  free(host);
  return 0;
}

int main(int argc, char** argv) {
  const int B = PB, S = PS, H = PH, HKV = PHKV, D = PD;          /* prefill */
  const int DB = DBSZ, DH = DHH, DHKV = DHKVV, L = DL;            /* decode, head_dim D */
  const float scale = SCALE;
  void *q, *k, *v, *pos, *cs, *sn, *out, *ws;
  void *dq, *kc, *vc, *lens, *qpos, *dcs, *dsn, *dout, *dws;
  size_t wsb, dwsb;
  int rc;
  if (argc < 2) return 1;
  snprintf(dir, sizeof dir, "%s", argv[1]);
  /* ---- prefill: q [B,S,H,D], k/v [B,S,HKV,D] bf16, positions [B,S] int64 */
  if ((rc = upload("q.bin", (size_t)B * S * H * D * 2, &q))) return rc;
  if ((rc = upload("k.bin", (size_t)B * S * HKV * D * 2, &k))) return rc;
  if ((rc = upload("v.bin", (size_t)B * S * HKV * D * 2, &v))) return rc;
  if ((rc = upload("pos.bin", (size_t)B * S * 8, &pos))) return rc;
  CK(cudaMalloc(&cs, (size_t)B * S * D * 4));
  CK(cudaMalloc(&sn, (size_t)B * S * D * 4));
  CK(cudaMalloc(&out, (size_t)B * S * H * D * 2));
  LA(llama_rope_table((const long long*)pos, B, S, D, 10000.0, 1.0, (float*)cs, (float*)sn, NULL));
  wsb = llama_attn_prefill_workspace_bytes(B, H, HKV, S, D, LLAMA_DT_BF16, 1);
  if (wsb == 0) return 7;
  CK(cudaMalloc(&ws, wsb));
  LA(llama_attn_prefill(q, k, v, (const float*)cs, (const float*)sn, B, H, HKV, S, D, scale, 1,
                        out, NULL, LLAMA_DT_BF16, ws, wsb, NULL));
  /* ---- decode: q [DB,DH,D], caches [DB,DHKV,L,D], lens [DB] int32, positions [DB] int64 */
  if ((rc = upload("dq.bin", (size_t)DB * DH * D * 2, &dq))) return rc;
  if ((rc = upload("kc.bin", (size_t)DB * DHKV * L * D * 2, &kc))) return rc;
  if ((rc = upload("vc.bin", (size_t)DB * DHKV * L * D * 2, &vc))) return rc;
  if ((rc = upload("lens.bin", (size_t)DB * 4, &lens))) return rc;
  if ((rc = upload("qpos.bin", (size_t)DB * 8, &qpos))) return rc;
  CK(cudaMalloc(&dcs, (size_t)DB * D * 4));
  CK(cudaMalloc(&dsn, (size_t)DB * D * 4));
  CK(cudaMalloc(&dout, (size_t)DB * DH * D * 2));
  LA(llama_rope_table((const long long*)qpos, DB, 1, D, 10000.0, 1.0, (float*)dcs, (float*)dsn,
                      NULL));
  dwsb = llama_attn_decode_workspace_bytes(DB, DH, L, D);
  CK(cudaMalloc(&dws, dwsb));
  LA(llama_attn_decode(dq, kc, vc, (const int*)lens, (const float*)dcs, (const float*)dsn, DB, DH,
                       DHKV, L, D, scale, dout, dws, dwsb, LLAMA_DT_BF16, NULL));
  CK(cudaDeviceSynchronize());
  LA(llama_attn_device_status(NULL));
  if ((rc = download("out.bin", out, (size_t)B * S * H * D * 2))) return rc;
  if ((rc = download("dout.bin", dout, (size_t)DB * DH * D * 2))) return rc;
  CK(cudaFree(q)); CK(cudaFree(k)); CK(cudaFree(v)); CK(cudaFree(pos)); CK(cudaFree(cs));
  CK(cudaFree(sn)); CK(cudaFree(out)); CK(cudaFree(ws)); CK(cudaFree(dq)); CK(cudaFree(kc));
  CK(cudaFree(vc)); CK(cudaFree(lens)); CK(cudaFree(qpos)); CK(cudaFree(dcs)); CK(cudaFree(dsn));
  CK(cudaFree(dout)); CK(cudaFree(dws));
  printf("ok\n");
  return 0;
}
"""


def _raw(t: torch.Tensor) -> bytes:
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        t = t.view(torch.int16)
    return t.numpy().tobytes()


def _bf16(path, shape):
    a = np.fromfile(path, dtype=np.uint16).astype(np.uint32) << 16
    return a.view(np.float32).astype(np.float64).reshape(shape)


def test_c_program_calls_prefill_and_decode_through_the_header(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    api.load()  # the in-tree library, built from the current sources
    B, S, H, HKV, D = 2, 200, 8, 2, 128
    DB, DHH, DHKVV, L = 3, 8, 2, 300
    scale = 1.0 / np.sqrt(D)
    cfg, x = W.small_prefill(B, S, H, HKV, D, torch.bfloat16, causal=True, seed=91)
    dcfg, y = W.small_decode(DB, DHH, DHKVV, D, L, torch.bfloat16, seed=92,
                             lens=torch.tensor([1, 150, 300], dtype=torch.int32))
    files = {"q.bin": x["q"], "k.bin": x["k"], "v.bin": x["v"], "pos.bin": x["pos"].to(torch.int64),
             "dq.bin": y["q"], "kc.bin": y["k_cache"], "vc.bin": y["v_cache"],
             "lens.bin": y["lens"].to(torch.int32), "qpos.bin": y["qpos"].to(torch.int64)}
    for name, t in files.items():
        (tmp_path / name).write_bytes(_raw(t))
    defs = dict(PB=B, PS=S, PH=H, PHKV=HKV, PD=D, DBSZ=DB, DHH=DHH, DHKVV=DHKVV, DL=L,
                SCALE=f"{scale:.9g}f")
    src = tmp_path / "boundary.c"
    src.write_text("".join(f"#define {k} {v}\n" for k, v in defs.items()) + PROGRAM)
    libdir = os.path.dirname(build.LIB)
    exe = tmp_path / "boundary"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", build.INCLUDE, "-isystem", os.path.join(CUDA, "include"), str(src),
                    "-L", libdir, "-lllama_attn", f"-Wl,-rpath,{libdir}",
                    "-L", os.path.join(CUDA, "lib64"), "-lcudart",
                    f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-o", str(exe)], check=True)
    run = subprocess.run([str(exe), str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert run.returncode == 0, run.stderr
    assert run.stdout.strip() == "ok"

    out = _bf16(tmp_path / "out.bin", (B, S, H * D))  # [b, S, H*D]: heads concatenated
    ref = oracle.prefill(x["q"], x["k"], x["v"], x["pos"], theta=cfg.theta, factor=cfg.factor,
                         scale=cfg.scale, causal=True)
    err = np.abs(out - ref.reshape(out.shape))
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())

    dout = _bf16(tmp_path / "dout.bin", (DB, DHH * D))
    dref = oracle.decode(y["q"], y["k_cache"], y["v_cache"], y["lens"], y["qpos"],
                         theta=dcfg.theta, factor=dcfg.factor, scale=dcfg.scale)
    derr = np.abs(dout - dref)
    assert np.all(np.isfinite(dout))
    assert derr.max() <= 2e-2 and derr.mean() <= 2e-3, (derr.max(), derr.mean())
