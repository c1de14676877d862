"""Host check (no GPU): the decode kernels' register counts, read from the
compiler's resource report (`-Xptxas -v`), stay inside the budgets their
launch plans rely on.

- In a chain of dependent layers, a CTA of the slab combine must fit on an SM
  beside a main-kernel CTA of the next layer (512 threads), so that the next
  layer's CTAs are resident early.  A combine of 78 registers broke this and
  measured q_proj 4.60 -> 5.24 us per layer.
- The rank-1 form runs two 512-thread CTAs per SM: at most 64 registers.

Registers are allocated per warp in multiples of 8 per thread; an SM holds
65536."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "boolean_weight_matmul_b200", "csrc", "gemv_lut.cu")
SM_REGISTERS = 65536


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


def _alloc(regs: int) -> int:
    return (regs + 7) // 8 * 8


@pytest.fixture(scope="module")
def registers(tmp_path_factory):
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not available")
    obj = str(tmp_path_factory.mktemp("regs") / "gemv_lut.o")
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-Xptxas", "-v", "-c", SRC, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    regs, current = {}, None
    for line in r.stderr.splitlines():
        m = re.search(r"Compiling entry function '(\w+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and current is not None:
            regs[current] = int(m.group(1))
            current = None
    assert regs, r.stderr[-2000:]
    return regs


def _pick(regs, pattern):
    found = {name: n for name, n in regs.items() if re.search(pattern, name)}
    assert found, f"no kernel matches {pattern}"
    return found


def test_combine_fits_beside_the_next_main_cta(registers):
    # gemv_lut8_kernel<K, XF32, SV = false>: mangled ...ILi<K>ELb<XF32>ELb0E...
    main = _pick(registers, r"gemv_lut8_kernelILi\dELb\dELb0E")
    multi = _pick(registers, r"gemv_lut8_multi_kernel")
    combine = _pick(registers, r"gemv_combine(_multi)?_kernel")
    worst_main = max(_alloc(n) for n in list(main.values()) + list(multi.values()))
    for name, n in combine.items():
        total = 512 * worst_main + 256 * _alloc(n)
        assert total <= SM_REGISTERS, f"{name}: {n} registers; with a {worst_main}-register main CTA: {total}"


def test_rank1_form_fits_two_ctas_per_sm(registers):
    sv = _pick(registers, r"gemv_lut8_kernelILi1ELb\dELb1E")
    for name, n in sv.items():
        assert 2 * 512 * _alloc(n) <= SM_REGISTERS, f"{name}: {n} registers"
