"""TEST INFRASTRUCTURE ONLY: assemble and compile a host-emulation binary for one kernel header.

The kernel header is copied next to sm100_stub.cuh (as sm100.cuh), emu.h and the harness, with
sm100_extracted.inc: the pure helpers cut from the real sm100.cuh (descriptor encoders and the
FMA-pipe exponential), so that the emulation restates no encoding of the library's own.
"""

from __future__ import annotations

import os
import re
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(os.path.dirname(HERE)), "exact_io_aware_77_b200", "csrc")
PURE_HELPERS = ("idesc_bf16_f32", "sw128_desc", "desc_advance", "exp2_poly_x2")
# headers whose every function the stub itself provides: the emulation gets an empty file
STUBBED_HEADERS = ("fp8_ops.cuh", "decode_ops.cuh")


def extract(src: str, name: str) -> str:
    """The full definition (signature line through its closing brace) of function `name`."""
    m = re.search(r"^[^\n]*\b" + re.escape(name) + r"\s*\(", src, re.M)
    if m is None:
        raise RuntimeError(f"{name} not found in sm100.cuh")
    i = src.index("{", m.end())
    depth = 0
    for j in range(i, len(src)):
        if src[j] == "{":
            depth += 1
        elif src[j] == "}":
            depth -= 1
            if depth == 0:
                return src[m.start():j + 1] + "\n"
    raise RuntimeError(f"unbalanced braces in {name}")


# Inline asm that a kernel header itself holds, replaced in the emulation's copy (only) by a
# call to the stub's stand-in.  The library's sources are not changed.
PATCHES = {
    "bwd_kernel.cuh": [
        (r'asm volatile\("cp\.async\.bulk\.shared::cluster\.global\.mbarrier::complete_tx::bytes.*?: "memory"\);',
         "emu_bulk_load(dst, src, bytes, bar);"),
    ],
}


def build(out_dir: str, kernel_header, harness: str, exe_name: str, defines=()) -> str:
    """kernel_header: one header name, or a list (a kernel header and the headers it includes)."""
    headers = [kernel_header] if isinstance(kernel_header, str) else list(kernel_header)
    # and every library header they include (sm100.cuh and the stubbed headers are the stub's)
    i = 0
    while i < len(headers):
        with open(os.path.join(CSRC, headers[i])) as f:
            for inc in re.findall(r'^#include "([^"/]+)"', f.read(), re.M):
                if inc not in headers and inc != "sm100.cuh" and inc not in STUBBED_HEADERS:
                    headers.append(inc)
        i += 1
    gxx = shutil.which("g++")
    if gxx is None:
        raise FileNotFoundError("g++")
    with open(os.path.join(CSRC, "sm100.cuh")) as f:
        real = f.read()
    with open(os.path.join(out_dir, "sm100_extracted.inc"), "w") as f:
        f.write("// cut from sm100.cuh by tests/host_emu/build_emu.py\n")
        for name in PURE_HELPERS:
            f.write(extract(real, name))
    for h in headers:
        with open(os.path.join(CSRC, h)) as f:
            text = f.read()
        for pattern, repl in PATCHES.get(h, []):
            text, n = re.subn(pattern, repl, text, flags=re.S)
            if n != 1:
                raise RuntimeError(f"patch for {h} matched {n} times")
        with open(os.path.join(out_dir, h), "w") as f:
            f.write(text)
    shutil.copy(os.path.join(HERE, "sm100_stub.cuh"), os.path.join(out_dir, "sm100.cuh"))
    for h in STUBBED_HEADERS:
        with open(os.path.join(out_dir, h), "w") as f:
            f.write("// provided by the host emulation's sm100.cuh\n#pragma once\n")
    shutil.copy(os.path.join(HERE, "emu.h"), os.path.join(out_dir, "emu.h"))
    shutil.copy(os.path.join(HERE, harness), os.path.join(out_dir, harness))
    exe = os.path.join(out_dir, exe_name)
    cmd = [gxx, "-std=c++20", "-O1", "-g", "-fsanitize=address,undefined", "-fno-sanitize-recover=all",
           "-fno-omit-frame-pointer", "-pthread"] + [f"-D{d}" for d in defines] + \
          ["-x", "c++", os.path.join(out_dir, harness), "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("host emulation does not compile:\n" + r.stderr[-6000:])
    return exe


def build_many(out_dir: str, jobs) -> dict:
    """Build several emulation binaries at once: jobs = {key: (kernel_header(s), harness, exe_name,
    defines)}; returns {key: path}.  The g++ runs overlap (they are independent processes)."""
    from concurrent.futures import ThreadPoolExecutor
    # each build gets its own directory, so the copies the builds write never collide
    with ThreadPoolExecutor(max_workers=min(4, len(jobs))) as pool:
        futures = {}
        for i, (key, (hdr, harness, exe, defines)) in enumerate(jobs.items()):
            sub = os.path.join(out_dir, f"b{i}")
            os.makedirs(sub, exist_ok=True)
            futures[key] = pool.submit(build, sub, hdr, harness, exe, defines)
        return {key: f.result() for key, f in futures.items()}
