"""CPU checks of the C-ABI library: it is built, it loads without a GPU, and
it exports every entry point that include/gca.h declares.  No compute call is
made here (that needs a GPU)."""
import os
import re
import subprocess

import pytest

from windowed_memory_attention_b200 import gca
from windowed_memory_attention_b200 import build as gbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gca.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gca_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def built():
    return gbuild.build()


def test_header_declares_the_five_calls():
    names = declared_functions()
    for call in ("gca_cache_create", "gca_append_frame", "gca_attend", "gca_evict_to_summary",
                 "gca_reset"):
        assert call in names


def test_library_loads_and_exports_every_declared_symbol(built):
    L = gca.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", built], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (gca_[a-z_]+)", out))
    assert set(declared_functions()) <= exported
    assert set(gca.EXPORTS) == set(declared_functions())


def test_status_strings(built):
    assert gca.gca_status_string(0) == "ok"
    assert "capacity" in gca.gca_status_string(2)
    assert gca.gca_status_string(99) == "unknown status"


def test_library_is_sm100a_only(built):
    # the kernels are compiled for sm_100a alone (no PTX fallback for other GPUs)
    assert "arch=compute_100a,code=sm_100a" in " ".join(gbuild.ARCH)


def test_create_without_gpu_fails_cleanly(built):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(gca.GCAError) as e:
        gca.gca_cache_create(num_layers=1, num_heads=2, image_tokens=16, num_anchor=3, window=4,
                             max_frames=32)
    assert e.value.name in ("GCA_ERR_INVALID_ARG", "GCA_ERR_CUDA")
