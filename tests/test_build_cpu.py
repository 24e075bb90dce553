"""The in-tree build decides by content whether an object or the library is current: an object is
redone when its source, a header or the flags changed, or when its recorded hash is missing or differs
(objects carried over from another checkout), and never because of a modification time alone."""
import os
import subprocess

import rank_latent_kv_vmla_b200.build as B


def _fake_toolchain(monkeypatch, tmp_path, compiled, links):
    csrc, inc = tmp_path / "csrc", tmp_path / "include"
    csrc.mkdir()
    inc.mkdir()
    for name, text in (("a.cu", "int a;"), ("b.cu", "int b;"), ("k.cuh", "#pragma once")):
        (csrc / name).write_text(text)
    (inc / "v.h").write_text("/* api */")
    monkeypatch.setattr(B, "CSRC", str(csrc))
    monkeypatch.setattr(B, "INCLUDE", str(inc))
    monkeypatch.setattr(B, "BUILD", str(tmp_path / "_build"))
    monkeypatch.setattr(B, "LIB", str(tmp_path / "libvmla.so"))

    def compile_(src, obj, extra):
        compiled.append(os.path.basename(src))
        with open(obj, "w") as f:
            f.write(open(src).read())
        return ""

    def run(cmd, **kw):
        if "--version" in cmd:
            return subprocess.CompletedProcess(cmd, 0, "nvcc fake\nrelease 0.0\n", "")
        out = cmd[cmd.index("-o") + 1]
        links.append(out)
        open(out, "w").close()
        return subprocess.CompletedProcess(cmd, 0, "", "")

    monkeypatch.setattr(B, "_compile", compile_)
    monkeypatch.setattr(B.subprocess, "run", run)
    monkeypatch.setattr(B, "nvcc", lambda: "nvcc")
    monkeypatch.setattr(B, "_NVCC_VERSION", [])
    return csrc, inc


def test_build_is_decided_by_content(monkeypatch, tmp_path):
    compiled, links = [], []
    csrc, inc = _fake_toolchain(monkeypatch, tmp_path, compiled, links)
    B.build()
    assert sorted(compiled) == ["a.cu", "b.cu"] and len(links) == 1
    del compiled[:], links[:]
    B.build()                                     # nothing changed
    assert compiled == [] and links == []
    later = os.path.getmtime(csrc / "a.cu") + 100
    os.utime(csrc / "a.cu", (later, later))       # a newer file with the same content
    B.build()
    assert compiled == [] and links == []
    (csrc / "a.cu").write_text("int a = 1;")      # a changed source: only its object, then the link
    B.build()
    assert compiled == ["a.cu"] and len(links) == 1
    del compiled[:], links[:]
    with open(os.path.join(B.BUILD, "b.o.sha256"), "w") as f:
        f.write("0" * 64)                         # an object whose record does not match
    B.build()
    assert compiled == ["b.cu"] and len(links) == 1
    del compiled[:], links[:]
    os.remove(B.LIB + ".sha256")                  # a library without a record is linked again
    B.build()
    assert compiled == [] and len(links) == 1
    del compiled[:], links[:]
    (inc / "v.h").write_text("/* api v2 */")      # a header change redoes every object
    B.build()
    assert sorted(compiled) == ["a.cu", "b.cu"] and len(links) == 1
